// The part of a block's exact selection that follows the scoring pass (pick.cuh has the
// selection itself and its page citations).  The scoring pass's last CTA has already taken
// the level-1 bin of the r-th smallest key and, when the pass predicted that bin, the
// exact threshold T.  Two grid-wide kernels do the rest, each returning at once when it
// has nothing to do:
//   - select_finish: when the bin was not predicted (rare; always for the first block),
//     re-read the region for the level-2 histogram of the chosen bin; the last CTA to
//     finish takes T;
//   - select_ties: when only some entries tied at T are taken, count the block's ties per
//     column over the grid; the last CTA finds the (column, row) cut-off.
// The level-2 histograms the block used are cleared by the row solve that follows.
#include "pick.cuh"

namespace pwp {
namespace {

// ctl without __restrict__: the last CTA's threads share decisions taken by one of them
// (through shared memory; see pick.cuh).
template <int SCORE>
__global__ void __launch_bounds__(pick::kThreads) select_finish_kernel(Ctl* ctl, Level2 l2,
                                                                      const float* __restrict__ W, int c, int b,
                                                                      int j, int q1,
                                                                      const float* __restrict__ sc, pwp_stats* st) {
  pdl_enter();
  __shared__ pick::Shared sh;
  if (cta_failed(st)) return;
  // the outcome of the scoring pass's last CTA (an earlier kernel)
  if (ctl->mode == 0 || ctl->l2_ready) return;
  const int tid = threadIdx.x;
  // the level-2 histogram of bin b1 over the region: rows over CTAs, columns over threads,
  // eight loads in flight per thread before their counts
  const unsigned int b1 = ctl->b1;
  const long long r1 = ctl->r1;
  constexpr int kU = 8;
  for (int r = blockIdx.x; r < c; r += gridDim.x) {
    const float* wr = W + (long long)r * b;
    for (int q0 = j + tid; q0 < q1; q0 += kU * blockDim.x) {
      float w[kU], p[kU];
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int q = q0 + u * blockDim.x;
        w[u] = q < q1 ? wr[q] : 0.f;
        p[u] = q < q1 ? __ldg(sc + q) : 0.f;
      }
#pragma unroll
      for (int u = 0; u < kU; ++u)
        if (q0 + u * blockDim.x < q1) count_level2(key_of<SCORE>(w[u], p[u]), b1, l2.reread, l2.reread_sum);
    }
  }
  if (!pick::last_cta(&ctl->ticket, sh)) return;
  pick::level2(ctl, l2, r1, 0, st, sh, 1, tid);
}

template <int SCORE>
__global__ void __launch_bounds__(pick::kThreads) select_ties_kernel(Ctl* ctl, Level2 l2,
                                                                    const float* __restrict__ W, int c, int b,
                                                                    int j, int j1, const float* __restrict__ sc,
                                                                    pwp_stats* st) {
  pdl_enter();
  __shared__ pick::Shared sh;
  if (cta_failed(st)) return;
  if (ctl->mode == 0 || !ctl->tie_scan) return;
  const unsigned int T = ctl->T;
  const long long m = ctl->m;
  const int gtid = blockIdx.x * blockDim.x + threadIdx.x, stride = gridDim.x * blockDim.x;
  pick::count_ties<SCORE>(T, l2, W, b, j, j1, sc, gtid >> 5, c, stride >> 5);
  if (!pick::last_cta(&ctl->ticket, sh)) return;
  pick::tie_cutoff<SCORE>(ctl, T, m, l2, W, c, b, j, j1, sc, sh, 1, threadIdx.x);
}

// ---------------------------------------------------------------- the stepwise sweep
// Rows sharded over ranks, the unstructured budget over all of them: the caller sums the
// histograms over ranks between these steps (see pwp_sweep_step).  hist1[kHist1Bins]
// carries this rank's removal count into the level-1 sum.

__global__ void publish_count_kernel(const Ctl* __restrict__ ctl, unsigned int* __restrict__ hist1,
                                     const pwp_stats* st) {
  pdl_enter();
  if (failed(st)) return;
  hist1[kHist1Bins] = (unsigned int)ctl->pruned;
}

__global__ void __launch_bounds__(pick::kThreads) pick_bin_kernel(Ctl* ctl, unsigned int* hist1,
                                                                  PickArgs pk, pwp_stats* st) {
  pdl_enter();
  __shared__ pick::Shared sh;
  if (cta_failed(st)) return;
  const long long pruned_all = (long long)hist1[kHist1Bins];   // summed over ranks
  pick::level1(ctl, hist1, pk.region_n, pk.global_budget, pk.quota, st, sh, 1, threadIdx.x,
               pk.global_budget ? pruned_all : -1);
  if (threadIdx.x == 0) hist1[kHist1Bins] = 0u;
}

template <int SCORE>
__global__ void __launch_bounds__(256) reread_kernel(const float* __restrict__ W, int c, int b, int q0, int q1,
                                                     const float* __restrict__ sc, const Ctl* __restrict__ ctl,
                                                     Level2 l2, const pwp_stats* st) {
  pdl_enter();
  if (cta_failed(st) || ctl->mode == 0 || ctl->l2_ready) return;
  const unsigned int b1 = ctl->b1;
  for (int r = blockIdx.x; r < c; r += gridDim.x) {
    const float* wr = W + (long long)r * b;
    for (int q = q0 + threadIdx.x; q < q1; q += blockDim.x)
      count_level2(key_of<SCORE>(wr[q], __ldg(sc + q)), b1, l2.reread, l2.reread_sum);
  }
}

__global__ void __launch_bounds__(pick::kThreads) pick_key_kernel(Ctl* ctl, Level2 l2, pwp_stats* st) {
  pdl_enter();
  __shared__ pick::Shared sh;
  if (cta_failed(st) || ctl->mode == 0) return;
  pick::level2(ctl, l2, (long long)ctl->r1, ctl->l2_ready, st, sh, 1, threadIdx.x);
}

template <int SCORE>
__global__ void __launch_bounds__(256) count_ties_kernel(const Ctl* __restrict__ ctl, Level2 l2,
                                                         const float* __restrict__ W, int c, int b, int j, int j1,
                                                         const float* __restrict__ sc, const pwp_stats* st) {
  pdl_enter();
  if (cta_failed(st) || ctl->mode == 0 || !ctl->tie_scan) return;
  const int gtid = blockIdx.x * blockDim.x + threadIdx.x, stride = gridDim.x * blockDim.x;
  pick::count_ties<SCORE>(ctl->T, l2, W, b, j, j1, sc, gtid >> 5, c, stride >> 5);
}

// The cut-off among tied entries when the rows are spread over ranks: (column, row) order
// with the rows of lower ranks first.  ties_all: every rank's per-column counts (world x
// kMaxBlock, this rank's own at `rank`).  This rank takes its tied entries in the columns
// before the cut-off column, none after it, and in it those that follow the lower ranks'.
template <int SCORE>
__global__ void __launch_bounds__(pick::kThreads) cut_ties_kernel(Ctl* ctl, Level2 l2, const float* __restrict__ W,
                                                                  int c, int b, int j, int j1,
                                                                  const float* __restrict__ sc,
                                                                  const unsigned int* __restrict__ ties_all,
                                                                  int world, int rank, pwp_stats* st) {
  pdl_enter();
  __shared__ pick::Shared sh;
  __shared__ long long s_pstar;
  if (cta_failed(st)) return;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (ctl->mode == 0 || !ctl->tie_scan) return;
  const int nJ = j1 - j;
  if (tid == 0) {
    const long long m = ctl->m;
    long long cum = 0, need = 0, before_me = 0, mine = 0;
    int qstar = -1;
    for (int qq = 0; qq < nJ && qstar < 0; ++qq) {
      long long cq = 0;
      for (int r = 0; r < world; ++r) cq += ties_all[(size_t)r * kMaxBlock + qq];
      if (cum + cq >= m) {
        qstar = qq;
        need = m - cum;
        for (int r = 0; r < rank; ++r) before_me += ties_all[(size_t)r * kMaxBlock + qq];
        mine = ties_all[(size_t)rank * kMaxBlock + qq];
      }
      cum += cq;
    }
    long long pstar = LLONG_MAX;                        // fewer than m ties: all are taken
    const long long local_need = need - before_me;
    sh.sel = -1;
    if (qstar >= 0) {
      if (local_need <= 0) pstar = (long long)qstar * c - 1;                  // none of this rank's
      else if (local_need >= mine) pstar = (long long)qstar * c + (c - 1);   // all of this rank's
      else sh.sel = qstar;                                                     // locate the row
    }
    sh.need = local_need;
    s_pstar = pstar;
  }
  __syncthreads();
  const int qstar = sh.sel;
  const long long need = sh.need;
  for (int i = tid; i < kMaxBlock; i += blockDim.x) l2.tie_count[i] = 0u;
  if (qstar >= 0) {
    const unsigned int T = ctl->T;
    const int q = j + qstar;
    const float scq = __ldg(sc + q);
    const int per = (c + pick::kThreads - 1) / pick::kThreads;
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
    __syncthreads();
    long long wbase = 0;
    for (int w = 0; w < warp; ++w) wbase += sh.warp[w];
    const long long bef = wbase + x - cnt;
    if (bef < need && need <= bef + cnt) {
      long long k = bef;
      for (int i = 0; i < per; ++i) {
        const int r = tid * per + i;
        if (r < c && key_of<SCORE>(W[(long long)r * b + q], scq) == T) {
          if (++k == need) {
            s_pstar = (long long)qstar * c + r;
            break;
          }
        }
      }
    }
  }
  __syncthreads();
  if (tid == 0) ctl->pstar = s_pstar;
}

}  // namespace

void launch_select_finish(int score, Ctl* ctl, Level2 l2, const float* W, int c, int b, int j, int j1, int q1,
                          const float* sc, pwp_stats* st, cudaStream_t s) {
  if (score == kWanda) {
    launch_pdl(select_finish_kernel<kWanda>, dim3(kNumSM), dim3(pick::kThreads), 0, s, ctl, l2, W, c, b, j, q1, sc,
               st);
    launch_pdl(select_ties_kernel<kWanda>, dim3(kNumSM), dim3(pick::kThreads), 0, s, ctl, l2, W, c, b, j, j1, sc, st);
  } else {
    launch_pdl(select_finish_kernel<kObs>, dim3(kNumSM), dim3(pick::kThreads), 0, s, ctl, l2, W, c, b, j, q1, sc, st);
    launch_pdl(select_ties_kernel<kObs>, dim3(kNumSM), dim3(pick::kThreads), 0, s, ctl, l2, W, c, b, j, j1, sc, st);
  }
}

}  // namespace pwp

namespace pwp {

// The stepwise sweep's selection steps (pwp_sweep_step): see the kernels above.
void launch_sweep_select(int step, int score, Ctl* ctl, unsigned int* hist1, Level2 l2, PickArgs pk, const float* W,
                         int c, int b, int j, int j1, int q1, const float* sc, const unsigned int* ties_all, int world,
                         int rank, pwp_stats* st, cudaStream_t s) {
  const bool wanda = score == kWanda;
  switch (step) {
    case 0:   // this rank's removal count into the level-1 sum
      launch_pdl(publish_count_kernel, dim3(1), dim3(1), 0, s, (const Ctl*)ctl, hist1, (const pwp_stats*)st);
      break;
    case 1:   // the level-1 bin from the summed histogram
      launch_pdl(pick_bin_kernel, dim3(1), dim3(pick::kThreads), 0, s, ctl, hist1, pk, st);
      break;
    case 2:   // this rank's level-2 counts of the chosen bin when it was not predicted
      if (wanda)
        launch_pdl(reread_kernel<kWanda>, dim3(min(c, 4 * kNumSM)), dim3(256), 0, s, W, c, b, j, q1, sc,
                   (const Ctl*)ctl, l2, (const pwp_stats*)st);
      else
        launch_pdl(reread_kernel<kObs>, dim3(min(c, 4 * kNumSM)), dim3(256), 0, s, W, c, b, j, q1, sc,
                   (const Ctl*)ctl, l2, (const pwp_stats*)st);
      break;
    case 3:   // the threshold from the summed level-2 histograms
      launch_pdl(pick_key_kernel, dim3(1), dim3(pick::kThreads), 0, s, ctl, l2, st);
      break;
    case 4:   // this rank's tied entries per block column
      if (wanda)
        launch_pdl(count_ties_kernel<kWanda>, dim3(kNumSM), dim3(256), 0, s, (const Ctl*)ctl, l2, W, c, b, j, j1, sc,
                   (const pwp_stats*)st);
      else
        launch_pdl(count_ties_kernel<kObs>, dim3(kNumSM), dim3(256), 0, s, (const Ctl*)ctl, l2, W, c, b, j, j1, sc,
                   (const pwp_stats*)st);
      break;
    case 5:   // this rank's cut-off among the ties, from every rank's counts
      if (wanda)
        launch_pdl(cut_ties_kernel<kWanda>, dim3(1), dim3(pick::kThreads), 0, s, ctl, l2, W, c, b, j, j1, sc,
                   ties_all, world, rank, st);
      else
        launch_pdl(cut_ties_kernel<kObs>, dim3(1), dim3(pick::kThreads), 0, s, ctl, l2, W, c, b, j, j1, sc,
                   ties_all, world, rank, st);
      break;
    default:
      break;
  }
}

}  // namespace pwp
