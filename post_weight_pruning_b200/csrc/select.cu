// The part of a block's exact selection that follows the scoring pass (pick.cuh has the
// selection itself and its page citations).  The scoring pass's last CTA has already taken
// the level-1 bin of the r-th smallest key and, when the pass predicted that bin, the
// exact threshold T.  One grid-wide kernel does the rest:
//   - when the bin was not predicted (rare): re-read the region for the level-2 histogram
//     of the chosen bin; the last CTA to finish takes T, and, if only some entries tied at
//     T are taken, counts the block's ties per column and finds the cut-off itself;
//   - otherwise, when only some tied entries are taken: count the block's ties per column
//     over the grid; the last CTA finds the (column, row) cut-off;
//   - and clears the level-2 histograms the block used, ready for the next block.
#include "pick.cuh"

namespace pwp {
namespace {

__device__ __forceinline__ void zero_words(unsigned int* p, int n, int first, int stride) {
  uint4* p4 = reinterpret_cast<uint4*>(p);
  const uint4 z = make_uint4(0u, 0u, 0u, 0u);
  for (int i = first; i < n / 4; i += stride) p4[i] = z;
}

template <int SCORE>
__global__ void __launch_bounds__(pick::kThreads) select_finish_kernel(Ctl* __restrict__ ctl, Level2 l2,
                                                                      const float* __restrict__ W, int c, int b,
                                                                      int j, int j1, int q1,
                                                                      const float* __restrict__ sc, pwp_stats* st) {
  pdl_enter();
  __shared__ pick::Shared sh;
  if (cta_failed(st)) return;
  const int tid = threadIdx.x;
  const int gtid = blockIdx.x * blockDim.x + tid, stride = gridDim.x * blockDim.x;
  const int mode = ctl->mode, ready = ctl->l2_ready, tie_scan = ctl->tie_scan;
  const bool dirty_pred = ctl->dirty_pred != 0;
  if (mode != 0 && !ready) {
    // the level-2 histogram of bin b1 over the region: rows over CTAs, columns over threads
    const unsigned int b1 = ctl->b1;
    for (int r = blockIdx.x; r < c; r += gridDim.x) {
      const float* wr = W + (long long)r * b;
      for (int q = j + tid; q < q1; q += blockDim.x)
        count_level2(key_of<SCORE>(wr[q], __ldg(sc + q)), b1, l2.reread, l2.reread_sum);
    }
    if (!pick::last_cta(&ctl->ticket, sh)) return;
    pick::level2(ctl, l2, st, sh, 1, tid);
    if (ctl->mode != 0 && ctl->tie_scan) {
      pick::count_ties<SCORE>(ctl, l2, W, b, j, j1, sc, tid >> 5, c, pick::kWarps);
      __threadfence_block();
      pick::sync(1);
      pick::tie_cutoff<SCORE>(ctl, l2, W, c, b, j, j1, sc, sh, 1, tid);
    }
    // this CTA alone clears what the block counted into
    if (dirty_pred) {
      zero_words(l2.pred, kHist2Bins, tid, blockDim.x);
      zero_words(l2.pred_sum, kHist2SumBins, tid, blockDim.x);
    }
    zero_words(l2.reread, kHist2Bins, tid, blockDim.x);
    zero_words(l2.reread_sum, kHist2SumBins, tid, blockDim.x);
    return;
  }
  // the predicted level-2 histogram was consumed by the scoring pass's last CTA
  if (dirty_pred) {
    zero_words(l2.pred, kHist2Bins, gtid, stride);
    zero_words(l2.pred_sum, kHist2SumBins, gtid, stride);
  }
  if (mode != 0 && tie_scan) {
    const int gwarp = gtid >> 5, nwarps = stride >> 5;
    pick::count_ties<SCORE>(ctl, l2, W, b, j, j1, sc, gwarp, c, nwarps);
    if (!pick::last_cta(&ctl->ticket, sh)) return;
    pick::tie_cutoff<SCORE>(ctl, l2, W, c, b, j, j1, sc, sh, 1, tid);
  }
}

}  // namespace

void launch_select_finish(int score, Ctl* ctl, Level2 l2, const float* W, int c, int b, int j, int j1, int q1,
                          const float* sc, pwp_stats* st, cudaStream_t s) {
  if (score == kWanda)
    launch_pdl(select_finish_kernel<kWanda>, dim3(kNumSM), dim3(pick::kThreads), 0, s, ctl, l2, W, c, b, j, j1, q1,
               sc, st);
  else
    launch_pdl(select_finish_kernel<kObs>, dim3(kNumSM), dim3(pick::kThreads), 0, s, ctl, l2, W, c, b, j, j1, q1,
               sc, st);
}

}  // namespace pwp
