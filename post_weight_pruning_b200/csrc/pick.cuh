// Exact selection of the r lowest-scoring weights of a region, as device functions run by
// 256 threads of one CTA (the last CTA of a grid-wide pass, found with an atomic ticket).
//
// "Pruning LLMs with Thanos", section "Contribution two: keep the budget global and the
// execution local", steps 1-4: the residual count r, the rescored active region, and
// exactly that many lowest-scoring weights as the candidate set.  For SparseGPT the region
// is the current block and r its quota.
//
// Keys are the bit patterns of the non-negative fp32 scores, so ordering keys orders
// scores.  The r-th smallest key T comes from a two-level radix select: a histogram of key
// bits [30:18] (level 1, built while the scores are produced) and one of bits [17:0] over
// the entries of the level-1 bin (level 2).  The threshold's level-1 bin rarely moves from
// one block to the next, so the scoring pass also builds the level-2 histogram of the
// previous block's bin; only when this block's bin differs is the region read again.  Among
// entries equal to T the order is (column, row) -- the pages fix none -- so when only some
// tied entries are taken, the cut-off position inside the current block is located too.
//
// One thread takes each decision and records it in the control block for later kernels;
// the CTA's other threads get it through shared memory (Shared), never by re-reading the
// control block, and the kernels that call these functions take their control-block and
// histogram pointers without __restrict__: a value written by one thread of a kernel and
// read by another through global memory must not be cached by the compiler across the
// barrier in between.
#pragma once

#include <climits>

#include "pwp_internal.cuh"

namespace pwp {
namespace pick {

constexpr int kThreads = 256, kWarps = kThreads / 32;

struct Shared {
  long long warp[kWarps];
  long long base;
  long long take;
  long long need;
  int sel;
  int last;
  // the decisions of the block's selection, for every thread of the CTA
  int mode;        // something is removed
  int ready;       // the predicted level-2 histogram holds the chosen bin
  int tie_scan;    // the cut-off among tied entries has to be located
  unsigned int T;  // the threshold key
  long long r1;    // rank of the take-th key inside the chosen level-1 bin
  long long m;     // entries tied at T that are taken
};

__device__ __forceinline__ long long warp_sum_ll(long long v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Named barrier over the kThreads participating threads.
__device__ __forceinline__ void sync(int bar) { asm volatile("bar.sync %0, %1;" ::"r"(bar), "r"(kThreads) : "memory"); }

// The bin of a histogram of NB bins holding the rank-th (1-based) entry, by threads
// 0..kThreads-1: while the range is wider than the thread count, each warp sums one
// kWarps-th of it (coalesced) and the range narrows to the slice holding the rank; the last
// range is resolved by a prefix sum, one bin per thread.  *bin = -1 when the histogram holds
// fewer entries; *before = the entries in lower bins.
template <int NB>
__device__ void find_rank(const unsigned int* __restrict__ hist, long long rank, int* bin, long long* before,
                          Shared& sh, int bar, int tid) {
  static_assert(NB >= kThreads && (NB & (NB - 1)) == 0, "power-of-two histogram");
  const int lane = tid & 31, warp = tid >> 5;
  int base = 0, size = NB;
  long long below = 0;
  while (size > kThreads) {
    const int per = size / kWarps;
    const unsigned int* h = hist + base + warp * per;
    long long sum = 0;
#pragma unroll 8
    for (int i = lane; i < per; i += 32) sum += h[i];   // eight loads in flight
    sum = warp_sum_ll(sum);
    if (lane == 0) sh.warp[warp] = sum;
    sync(bar);
    if (tid == 0) {
      long long cum = 0;
      int sel = -1;
      for (int w = 0; w < kWarps; ++w) {
        if (rank - below > cum && rank - below <= cum + sh.warp[w]) { sel = w; break; }
        cum += sh.warp[w];
      }
      sh.sel = sel;
      sh.base = cum;
    }
    sync(bar);
    const int sel = sh.sel;
    const long long cum = sh.base;
    sync(bar);   // the shared words are rewritten next
    if (sel < 0) {
      *bin = -1;
      *before = 0;
      return;
    }
    base += sel * per;
    below += cum;
    size = per;
  }
  const long long v = tid < size ? (long long)hist[base + tid] : 0;
  long long x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const long long y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) sh.warp[warp] = x;
  if (tid == 0) sh.sel = -1;
  sync(bar);
  long long wbase = 0;
  for (int w = 0; w < warp; ++w) wbase += sh.warp[w];
  const long long incl = below + wbase + x;
  if (v > 0 && rank > incl - v && rank <= incl) {   // exactly one thread when 1 <= rank <= total
    sh.sel = base + tid;
    sh.base = incl - v;
  }
  sync(bar);
  const int sel = sh.sel;
  const long long bef = sh.base;
  sync(bar);
  *bin = sel;
  *before = sel < 0 ? 0 : bef;
}

// N words from global into shared memory by threads 0..kThreads-1, every load issued before
// the first store, then the named barrier.
template <int N>
__device__ __forceinline__ void stage_words(unsigned int* dst, const unsigned int* src, int bar, int tid) {
  static_assert(N % kThreads == 0, "whole rounds");
  unsigned int v[N / kThreads];
#pragma unroll
  for (int k = 0; k < N / kThreads; ++k) v[k] = src[tid + kThreads * k];
#pragma unroll
  for (int k = 0; k < N / kThreads; ++k) dst[tid + kThreads * k] = v[k];
  sync(bar);
}

// Step 1 of the budget loop and the level-1 bin: take = min(r, region) with r the residual
// global count (Thanos) or the block quota (SparseGPT); the bin of the take-th key; whether
// the scoring pass predicted it (then the level-2 histogram is ready).  Clears the level-1
// histogram for the next pass.
// (pruned: the removals so far over every row the budget counts; -1 for this call's own.)
// On return sh.mode, sh.ready and sh.r1 hold the outcome for every thread.
__device__ inline void level1(Ctl* ctl, unsigned int* hist1, long long region_n, int global_budget,
                              long long quota, pwp_stats* st, Shared& sh, int bar, int tid, long long pruned = -1,
                              const unsigned int* staged = nullptr) {
  if (tid == 0) {
    const long long r = global_budget ? ctl->zstar - (pruned >= 0 ? pruned : ctl->pruned) : quota;
    long long take = r < region_n ? r : region_n;
    if (take < r) st->shortfall = 1;
    if (take < 0) take = 0;
    ctl->take = take;
    ctl->mode = take > 0 ? 1 : 0;
    ctl->l2_ready = 0;
    ctl->dirty_pred = ctl->b1_valid;   // the scoring pass counted into the predicted histogram
    ctl->dirty_reread = 0;
    ctl->tie_scan = 0;
    sh.take = take;
    sh.mode = take > 0 ? 1 : 0;
    sh.ready = 0;
    sh.tie_scan = 0;
    sh.r1 = 0;
  }
  sync(bar);
  const long long take = sh.take;
  if (take > 0) {
    int bin;
    long long before;
    find_rank<kHist1Bins>(staged ? staged : hist1, take, &bin, &before, sh, bar, tid);
    if (tid == 0) {
      if (bin < 0) {
        set_error(st, PWP_EBUDGET, kSitePick);
        ctl->mode = 0;
        sh.mode = 0;
      } else {
        const bool hit = ctl->b1_valid && ctl->b1 == (unsigned int)bin;
        ctl->l2_ready = hit ? 1 : 0;
        ctl->dirty_reread = hit ? 0 : 1;
        if (!hit) st->reread_blocks += 1;
        ctl->b1 = (unsigned int)bin;
        ctl->b1_valid = 1;
        ctl->r1 = (unsigned int)(take - before);
        ctl->count_less = before;
        sh.ready = hit ? 1 : 0;
        sh.r1 = take - before;
      }
    }
  }
  sync(bar);
  for (int i = tid; i < kHist1Bins; i += kThreads) hist1[i] = 0u;
}

// The exact key T from the level-2 histogram of the chosen level-1 bin (the predicted one
// when `ready`, else the re-read one), the number m of entries tied at T that are taken,
// and whether the cut-off among the ties has to be located.  r1: the rank inside the bin
// (level1's sh.r1, or the control block's when level1 ran in an earlier kernel).  On
// return sh.mode, sh.T, sh.m and sh.tie_scan hold the outcome for every thread.
__device__ inline void level2(Ctl* ctl, Level2 l2, long long r1, int ready, pwp_stats* st, Shared& sh, int bar,
                              int tid, unsigned int* stage = nullptr) {
  const unsigned int* h2 = ready ? l2.pred : l2.reread;
  const unsigned int* h2s = ready ? l2.pred_sum : l2.reread_sum;
  int sb;
  long long before_s;
  if (stage) {
    // the summary and then the chosen summary bin's counts go through shared memory, each
    // with all its loads in flight (a rank search over global memory pays an L2 round trip
    // per narrowing step)
    stage_words<kHist2SumBins>(stage, h2s, bar, tid);
    find_rank<kHist2SumBins>(stage, r1, &sb, &before_s, sh, bar, tid);
  } else {
    find_rank<kHist2SumBins>(h2s, r1, &sb, &before_s, sh, bar, tid);
  }
  int sub = -1;
  long long before_sub = 0;
  if (sb >= 0) {
    const unsigned int* hsub = h2 + ((size_t)sb << kHist2SumShift);
    if (stage) {
      stage_words<(1 << kHist2SumShift)>(stage + kHist2SumBins, hsub, bar, tid);
      hsub = stage + kHist2SumBins;
    }
    find_rank<(1 << kHist2SumShift)>(hsub, r1 - before_s, &sub, &before_sub, sh, bar, tid);
  }
  if (sb < 0 || sub < 0) {
    if (tid == 0) {
      set_error(st, PWP_EBUDGET, kSitePick);
      ctl->mode = 0;
      sh.mode = 0;
      sh.tie_scan = 0;
    }
    sync(bar);
    return;
  }
  if (tid == 0) {
    const int lo = (sb << kHist2SumShift) + sub;
    const long long ties = h2[lo];
    const long long count_less = ctl->count_less + before_s + before_sub;
    const long long m = ctl->take - count_less;   // 1 <= m <= ties
    const unsigned int T = (ctl->b1 << kKeyLoBits) | (unsigned int)lo;
    const int tie_scan = m < ties ? 1 : 0;        // some but not all tied entries are taken
    ctl->T = T;
    ctl->ties = ties;
    ctl->m = m;
    ctl->count_less = count_less;
    ctl->pstar = LLONG_MAX;
    if (ties > 1) st->tie_blocks += 1;
    ctl->tie_scan = tie_scan;
    sh.mode = 1;
    sh.T = T;
    sh.m = m;
    sh.tie_scan = tie_scan;
  }
  sync(bar);
}

// Counts, per block column, of the block's entries whose key equals T, over the rows
// [r_begin, r_end) with stride r_step, added to tie_count (lane l: columns l + 32e).
template <int SCORE>
__device__ inline void count_ties(unsigned int T, Level2 l2, const float* W, int b, int j, int j1,
                                  const float* __restrict__ sc, int r_begin, int r_end, int r_step) {
  const int nJ = j1 - j, lane = threadIdx.x & 31;
  constexpr int E = kMaxBlock / 32;
  unsigned int cnt[E];
  float scv[E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    cnt[e] = 0u;
    scv[e] = lane + 32 * e < nJ ? __ldg(sc + j + lane + 32 * e) : 0.f;
  }
  for (int row = r_begin; row < r_end; row += r_step) {
    const float* wr = W + (long long)row * b + j;
#pragma unroll
    for (int e = 0; e < E; ++e)
      if (lane + 32 * e < nJ && key_of<SCORE>(wr[lane + 32 * e], scv[e]) == T) ++cnt[e];
  }
#pragma unroll
  for (int e = 0; e < E; ++e)
    if (cnt[e]) red_add_global(&l2.tie_count[lane + 32 * e], cnt[e]);
}

// The cut-off among the tied entries: with m of them taken in (column, row) order, the
// column holding the m-th, then its row (the threads scan that column); the per-column
// counts are zeroed for the next block.
template <int SCORE>
__device__ inline void tie_cutoff(Ctl* ctl, unsigned int T, long long m, Level2 l2, const float* W, int c, int b,
                                  int j, int j1, const float* __restrict__ sc, Shared& sh, int bar, int tid) {
  const int lane = tid & 31, warp = tid >> 5;
  const int nJ = j1 - j;
  {
    // the column holding the m-th tied entry, by a prefix sum of the per-column counts
    // (one column per thread; the first column whose running count reaches m)
    const long long cq = tid < nJ ? (long long)l2.tie_count[tid] : 0;
    long long x = cq;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long yv = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += yv;
    }
    if (lane == 31) sh.warp[warp] = x;
    if (tid == 0) sh.sel = -1;   // no such column: fewer than m ties inside the block
    sync(bar);
    long long incl = x;
    for (int w = 0; w < warp; ++w) incl += sh.warp[w];
    if (cq > 0 && incl >= m && incl - cq < m) {
      sh.sel = tid;
      sh.need = m - (incl - cq);   // 1-based rank of the last taken tie inside that column
    }
    sync(bar);
  }
  const int qstar = sh.sel;
  const long long need = sh.need;
  sync(bar);
  for (int i = tid; i < kMaxBlock; i += kThreads) l2.tie_count[i] = 0u;
  if (qstar < 0) return;   // fewer than m ties inside the block: all of them are taken
  const int q = j + qstar;
  const float scq = __ldg(sc + q);
  const int per = (c + kThreads - 1) / kThreads;
  long long cnt = 0;
  for (int i = 0; i < per; ++i) {
    const int r = tid * per + i;
    if (r < c && key_of<SCORE>(W[(long long)r * b + q], scq) == T) ++cnt;
  }
  long long x = cnt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const long long yv = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += yv;
  }
  if (lane == 31) sh.warp[warp] = x;
  sync(bar);
  long long wbase = 0;
  for (int w = 0; w < warp; ++w) wbase += sh.warp[w];
  const long long bef = wbase + x - cnt;
  if (bef < need && need <= bef + cnt) {
    long long k = bef;
    for (int i = 0; i < per; ++i) {
      const int r = tid * per + i;
      if (r < c && key_of<SCORE>(W[(long long)r * b + q], scq) == T) {
        if (++k == need) {
          ctl->pstar = (long long)qstar * c + r;
          break;
        }
      }
    }
  }
  sync(bar);
}

// True in exactly one CTA of the grid: the last to arrive, once every CTA's earlier global
// writes (histogram counts) are visible to it.  Called by all threads of the CTA after its
// last global write; the counter is reset for its next use.
__device__ inline bool last_cta(unsigned int* ticket, Shared& sh) {
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    const unsigned int t = atomicAdd(ticket, 1u);
    sh.last = (t == gridDim.x - 1) ? 1 : 0;
    if (sh.last) *ticket = 0u;
  }
  __syncthreads();
  if (sh.last) __threadfence();
  return sh.last != 0;
}

// After a scoring pass (all CTAs have added their level-1 counts): the last CTA takes the
// level-1 bin and, when the predicted level-2 histogram holds, the exact threshold.
// stage: kHist1Bins words of shared memory the CTA no longer needs, through which the rank
// searches read their histograms (or nullptr: straight from global memory).
__device__ inline void after_scoring(Ctl* ctl, unsigned int* hist1, Level2 l2, long long region_n,
                                     int global_budget, long long quota, pwp_stats* st, Shared& sh,
                                     unsigned int* stage = nullptr) {
  if (!last_cta(&ctl->ticket, sh)) return;
  const int tid = threadIdx.x;
  if (tid >= kThreads) return;
  if (failed(st)) {
    for (int i = tid; i < kHist1Bins; i += kThreads) hist1[i] = 0u;
    return;
  }
  if (stage) stage_words<kHist1Bins>(stage, hist1, 1, tid);
  level1(ctl, hist1, region_n, global_budget, quota, st, sh, 1, tid, -1, stage);
  if (sh.mode != 0 && sh.ready) level2(ctl, l2, sh.r1, 1, st, sh, 1, tid, stage);
}

}  // namespace pick
}  // namespace pwp
