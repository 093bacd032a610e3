// Exact selection of the r lowest-scoring weights of a region.
//
// "Pruning LLMs with Thanos", section "Contribution two: keep the budget global and
// the execution local", steps 1-4: the residual count r, the rescored active region,
// and "exactly that many lowest-scoring weights" as the candidate set.  For SparseGPT
// the region is the current block and r its quota.
//
// Keys are the bit patterns of the non-negative fp32 scores, so ordering keys orders
// scores.  The r-th smallest key T is found by a two-level radix select:
//   level 1: a histogram of key bits [30:18] (built while the scores are produced),
//   level 2: a histogram of bits [17:0] over the entries of the level-1 bin,
// then T = (bin1 << 18) | bin2.  The threshold's level-1 bin rarely moves from one block
// to the next, so the scoring pass also builds the level-2 histogram of the previous
// block's bin; only when this block's bin differs is the region read again (refine).  Among entries equal to T, the order is (column, row)
// -- the pages do not fix one -- so when only some tied entries are taken, the cut-off
// position inside the current block is located as well.
#include <climits>

#include "pwp_internal.cuh"

namespace pwp {
namespace {

__device__ __forceinline__ long long warp_sum_ll(long long v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Find, in a histogram of NB bins (1024 threads), the bin holding the `rank`-th
// (1-based) entry.  While the range is wider than the CTA, each of the 32 warps sums
// one 32nd of it (coalesced) and the range narrows to the warp slice holding the rank;
// the last range (at most 1024 bins) is resolved by a CTA-wide prefix sum.  Returns
// the bin in *bin (-1 if the histogram holds fewer entries) and the number of entries
// in lower bins in *before.
template <int NB>
__device__ void find_rank(const unsigned int* __restrict__ hist, long long rank, int* bin,
                          long long* before, long long* sh_warp, int* sh_sel, long long* sh_base) {
  static_assert(NB >= 32 && (NB & (NB - 1)) == 0, "power-of-two histogram");
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int base = 0;
  int size = NB;
  long long below = 0;
  while (size > 1024) {
    const int per = size / 32;
    const unsigned int* h = hist + base + warp * per;
    long long sum = 0;
    for (int i = lane; i < per; i += 32) sum += h[i];
    sum = warp_sum_ll(sum);
    if (lane == 0) sh_warp[warp] = sum;
    __syncthreads();
    if (tid == 0) {
      long long cum = 0;
      int sel = -1;
      for (int w = 0; w < 32; ++w) {
        if (rank - below > cum && rank - below <= cum + sh_warp[w]) { sel = w; break; }
        cum += sh_warp[w];
      }
      *sh_sel = sel;
      *sh_base = cum;
    }
    __syncthreads();
    const int sel = *sh_sel;
    const long long cum = *sh_base;
    __syncthreads();  // sh_warp / sh_sel are rewritten by the next round
    if (sel < 0) {
      *bin = -1;
      *before = 0;
      return;
    }
    base += sel * per;
    below += cum;
    size = per;
  }
  // last range: one bin per thread, inclusive prefix over the CTA
  const long long v = tid < size ? (long long)hist[base + tid] : 0;
  long long x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const long long y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) sh_warp[warp] = x;
  if (tid == 0) *sh_sel = -1;
  __syncthreads();
  long long wbase = 0;
  for (int w = 0; w < warp; ++w) wbase += sh_warp[w];
  const long long incl = below + wbase + x;
  // exactly one thread holds the rank when 1 <= rank <= total
  if (v > 0 && rank > incl - v && rank <= incl) {
    *sh_sel = base + tid;
    *sh_base = incl - v;
  }
  __syncthreads();
  const int sel = *sh_sel;
  const long long bef = *sh_base;
  __syncthreads();  // the caller reuses the shared words
  *bin = sel;
  *before = sel < 0 ? 0 : bef;
}

__global__ void __launch_bounds__(1024) pick1_kernel(Ctl* ctl, unsigned int* __restrict__ hist1, long long region_n,
                                                     int global_budget, long long quota, pwp_stats* st) {
  pdl_enter();
  __shared__ long long sh_warp[32];
  __shared__ int sh_sel;
  __shared__ long long sh_base, s_take;
  if (cta_failed(st)) return;
  if (threadIdx.x == 0) {
    long long r = global_budget ? ctl->zstar - ctl->pruned : quota;
    long long take = r < region_n ? r : region_n;
    if (take < r) st->shortfall = 1;
    if (take < 0) take = 0;
    ctl->take = take;
    ctl->mode = take > 0 ? 1 : 0;
    ctl->l2_ready = 0;
    ctl->dirty_pred = ctl->b1_valid;  // the scoring pass counted into the predicted histogram
    ctl->dirty_reread = 0;
    ctl->tie_scan = 0;
    s_take = take;
  }
  __syncthreads();
  const long long take = s_take;
  if (take > 0) {
    int bin;
    long long before;
    find_rank<kHist1Bins>(hist1, take, &bin, &before, sh_warp, &sh_sel, &sh_base);
    if (threadIdx.x == 0) {
      if (bin < 0) {
        set_error(st, PWP_EBUDGET, kSitePick);
        ctl->mode = 0;
      } else {
        const bool hit = ctl->b1_valid && ctl->b1 == (unsigned int)bin;
        ctl->l2_ready = hit ? 1 : 0;
        ctl->dirty_reread = hit ? 0 : 1;
        if (!hit) st->reread_blocks += 1;
        ctl->b1 = (unsigned int)bin;
        ctl->b1_valid = 1;
        ctl->r1 = (unsigned int)(take - before);
        ctl->count_less = before;
      }
    }
    __syncthreads();
  }
  for (int i = threadIdx.x; i < kHist1Bins; i += blockDim.x) hist1[i] = 0u;
}

// Level-2 histogram (re-read): the low kKeyLoBits key bits of the entries whose top
// bits equal b1, when the scoring pass predicted another bin.  One row per CTA
// iteration, columns across threads (coalesced).
template <int SCORE>
__global__ void __launch_bounds__(256) refine_kernel(const float* __restrict__ W, int c, int b, int q0,
                                                     int q1, const float* __restrict__ sc,
                                                     const Ctl* __restrict__ ctl, unsigned int* __restrict__ h2,
                                                     unsigned int* __restrict__ h2s, const pwp_stats* st) {
  pdl_enter();
  if (cta_failed(st) || ctl->mode == 0 || ctl->l2_ready) return;
  const unsigned int b1 = ctl->b1;
  for (int r = blockIdx.x; r < c; r += gridDim.x) {
    const float* wr = W + (long long)r * b;
    for (int q = q0 + threadIdx.x; q < q1; q += blockDim.x)
      count_level2(key_of<SCORE>(wr[q], __ldg(sc + q)), b1, h2, h2s);
  }
}

__global__ void __launch_bounds__(1024) pick2_kernel(Ctl* ctl, Level2 l2, pwp_stats* st) {
  pdl_enter();
  __shared__ long long sh_warp[32];
  __shared__ int sh_sel;
  __shared__ long long sh_base;
  if (cta_failed(st) || ctl->mode == 0) return;
  const int tid = threadIdx.x;
  const long long r1 = ctl->r1;
  const unsigned int* h2 = ctl->l2_ready ? l2.pred : l2.reread;
  const unsigned int* h2s = ctl->l2_ready ? l2.pred_sum : l2.reread_sum;
  // summary bin first, then the 512 level-2 bins under it
  int sb;
  long long before_s;
  find_rank<kHist2SumBins>(h2s, r1, &sb, &before_s, sh_warp, &sh_sel, &sh_base);
  int sub = -1;
  long long before_sub = 0;
  if (sb >= 0)
    find_rank<(1 << kHist2SumShift)>(h2 + ((size_t)sb << kHist2SumShift), r1 - before_s, &sub, &before_sub,
                                     sh_warp, &sh_sel, &sh_base);
  if (sb < 0 || sub < 0) {
    if (tid == 0) set_error(st, PWP_EBUDGET, kSitePick);
    return;
  }
  const int lo = (sb << kHist2SumShift) + sub;
  const long long before2 = before_s + before_sub;
  const unsigned int T = (ctl->b1 << kKeyLoBits) | (unsigned int)lo;
  const long long ties = h2[lo];
  const long long count_less = ctl->count_less + before2;
  const long long m = ctl->take - count_less;  // 1 <= m <= ties
  __syncthreads();
  if (tid == 0) {
    ctl->T = T;
    ctl->ties = ties;
    ctl->m = m;
    ctl->count_less = count_less;
    ctl->pstar = LLONG_MAX;
    if (ties > 1) st->tie_blocks += 1;
  }
  // some but not all tied entries are taken: the grid-wide count and the cut-off search follow
  if (tid == 0) ctl->tie_scan = m < ties ? 1 : 0;
}

// Zero the level-2 histograms this block wrote, ready for the next block; and, when only
// some of the entries tied at T are taken, count the block's tied entries per column
// (rows over the grid's warps, lane l counting columns l + 32e in registers).
template <int SCORE>
__global__ void __launch_bounds__(256) clear_level2_kernel(const Ctl* __restrict__ ctl, Level2 l2,
                                                           const float* __restrict__ W, int c, int b, int j, int j1,
                                                           const float* __restrict__ sc) {
  pdl_enter();
  const bool a = ctl->dirty_pred != 0, r = ctl->dirty_reread != 0;
  const int gtid = blockIdx.x * blockDim.x + threadIdx.x, stride = gridDim.x * blockDim.x;
  if (a || r) {
    uint4* pa = reinterpret_cast<uint4*>(l2.pred);
    uint4* pr = reinterpret_cast<uint4*>(l2.reread);
    const uint4 z = make_uint4(0u, 0u, 0u, 0u);
    for (int i = gtid; i < kHist2Bins / 4; i += stride) {
      if (a) pa[i] = z;
      if (r) pr[i] = z;
    }
    for (int i = gtid; i < kHist2SumBins; i += stride) {
      if (a) l2.pred_sum[i] = 0u;
      if (r) l2.reread_sum[i] = 0u;
    }
  }
  if (ctl->mode == 0 || !ctl->tie_scan) return;
  const unsigned int T = ctl->T;
  const int nJ = j1 - j, lane = threadIdx.x & 31;
  const int gwarp = gtid >> 5, nwarps = stride >> 5;
  constexpr int E = kMaxBlock / 32;
  unsigned int cnt[E];
  float scv[E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    cnt[e] = 0u;
    scv[e] = lane + 32 * e < nJ ? __ldg(sc + j + lane + 32 * e) : 0.f;
  }
  for (int row = gwarp; row < c; row += nwarps) {
    const float* wr = W + (long long)row * b + j;
    float v[E];
#pragma unroll
    for (int e = 0; e < E; ++e) v[e] = lane + 32 * e < nJ ? wr[lane + 32 * e] : 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e)
      if (lane + 32 * e < nJ && key_of<SCORE>(v[e], scv[e]) == T) ++cnt[e];
  }
#pragma unroll
  for (int e = 0; e < E; ++e)
    if (cnt[e]) atomicAdd(&l2.tie_count[lane + 32 * e], cnt[e]);
}

// The cut-off among the tied entries: with m of them taken in (column, row) order, the
// column holding the m-th, then its row (one CTA scans that column); the per-column
// counts are zeroed for the next block.
template <int SCORE>
__global__ void __launch_bounds__(1024) tie_pick_kernel(Ctl* ctl, Level2 l2, const float* __restrict__ W, int c,
                                                        int b, int j, int j1, const float* __restrict__ sc,
                                                        pwp_stats* st) {
  pdl_enter();
  __shared__ long long sh_warp[32];
  __shared__ int s_qstar;
  __shared__ long long s_need;
  if (cta_failed(st) || ctl->mode == 0 || !ctl->tie_scan) return;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nJ = j1 - j;
  const unsigned int T = ctl->T;
  const long long m = ctl->m;
  if (tid == 0) {
    long long cum = 0;
    int qstar = -1;
    for (int qq = 0; qq < nJ; ++qq) {
      const long long cq = l2.tie_count[qq];
      if (cum + cq >= m) { qstar = qq; break; }
      cum += cq;
    }
    s_qstar = qstar;
    s_need = m - cum;  // 1-based rank of the last taken tie inside column qstar
  }
  __syncthreads();
  for (int i = tid; i < kMaxBlock; i += blockDim.x) l2.tie_count[i] = 0u;
  if (s_qstar < 0) return;  // fewer than m ties inside the block: all of them are taken
  const int q = j + s_qstar;
  const float scq = __ldg(sc + q);
  const int per = (c + 1023) / 1024;
  long long cnt = 0;
  for (int i = 0; i < per; ++i) {
    const int r = tid * per + i;
    if (r < c && key_of<SCORE>(W[(long long)r * b + q], scq) == T) ++cnt;
  }
  // exclusive scan of cnt over the CTA
  long long x = cnt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const long long yv = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += yv;
  }
  if (lane == 31) sh_warp[warp] = x;
  __syncthreads();
  long long wbase = 0;
  for (int w = 0; w < warp; ++w) wbase += sh_warp[w];
  const long long bef = wbase + x - cnt;
  const long long need = s_need;
  if (bef < need && need <= bef + cnt) {
    long long k = bef;
    for (int i = 0; i < per; ++i) {
      const int r = tid * per + i;
      if (r < c && key_of<SCORE>(W[(long long)r * b + q], scq) == T) {
        if (++k == need) {
          ctl->pstar = (long long)s_qstar * c + r;
          break;
        }
      }
    }
  }
}

}  // namespace

void launch_pick1(Ctl* ctl, unsigned int* hist1, long long region_n, int global_budget, long long quota,
                  pwp_stats* st, cudaStream_t s) {
  launch_pdl(pick1_kernel, dim3(1), dim3(1024), 0, s, ctl, hist1, region_n, global_budget, quota, st);
}

void launch_refine(int score, const float* W, int c, int b, int q0, int q1, const float* sc,
                   const Ctl* ctl, Level2 l2, const pwp_stats* st, cudaStream_t s) {
  const int grid = c < 4 * kNumSM ? c : 4 * kNumSM;
  if (score == kWanda)
    launch_pdl(refine_kernel<kWanda>, dim3(grid), dim3(256), 0, s, W, c, b, q0, q1, sc, ctl, l2.reread, l2.reread_sum, st);
  else
    launch_pdl(refine_kernel<kObs>, dim3(grid), dim3(256), 0, s, W, c, b, q0, q1, sc, ctl, l2.reread, l2.reread_sum, st);
}

void launch_pick2(Ctl* ctl, Level2 l2, pwp_stats* st, cudaStream_t s) {
  launch_pdl(pick2_kernel, dim3(1), dim3(1024), 0, s, ctl, l2, st);
}

void launch_clear_level2(int score, const Ctl* ctl, Level2 l2, const float* W, int c, int b, int j, int j1,
                         const float* sc, cudaStream_t s) {
  if (score == kWanda)
    launch_pdl(clear_level2_kernel<kWanda>, dim3(kNumSM), dim3(256), 0, s, ctl, l2, W, c, b, j, j1, sc);
  else
    launch_pdl(clear_level2_kernel<kObs>, dim3(kNumSM), dim3(256), 0, s, ctl, l2, W, c, b, j, j1, sc);
}

void launch_tie_pick(int score, Ctl* ctl, Level2 l2, const float* W, int c, int b, int j, int j1, const float* sc,
                     pwp_stats* st, cudaStream_t s) {
  if (score == kWanda)
    launch_pdl(tie_pick_kernel<kWanda>, dim3(1), dim3(1024), 0, s, ctl, l2, W, c, b, j, j1, sc, st);
  else
    launch_pdl(tie_pick_kernel<kObs>, dim3(1), dim3(1024), 0, s, ctl, l2, W, c, b, j, j1, sc, st);
}

}  // namespace pwp
