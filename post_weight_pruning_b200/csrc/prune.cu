// Block sweep of the layer prune: scoring, exact mask selection, per-row solves and
// the trailing compensation update.
//
// "Pruning LLMs with Thanos":
//   - section "Contribution one: solve a selected set directly": for a row with
//     selected set Q in the current block, u = W[Q], R = K[Q, A], R-hat = K[Q, Q] with
//     K the active inverse Hessian; delta = -u^T R-hat^-1 R.
//   - section "Contribution two: keep the budget global and the execution local":
//     residual count, rescoring of the whole active region with activation-aware
//     scores, the r lowest as candidates, intersection with the block, solve,
//     decrement.
//   - N:M: local group masks, same joint solve (last paragraph of that section).
// "Weight Pruning in Large Language Models ..." (llms.blog), section "SparseGPT":
//   column-sequential OBS update W[:, q+1:] -= (W_q / [H^-1]_qq) H^-1[q, q+1:].
//
// With U upper and H_d^-1 = U^T U, the active inverse for block J = [j, j+B) and
// A = [j, b) is K[J, A] = U[J,J]^T U[J,A].  So the row update is
//   delta_k = -(U_JJ z_k)^T U[J, A],  z_k = R-hat^-1 u,  R-hat = Hb[Q,Q], Hb = U_JJ^T U_JJ,
// which splits into an in-block part (Hb rows) and a rank-B trailing update
// W[:, j+B:] -= Z' U[J, j+B:] with Z'_k = U_JJ z_k.  The trailing update of block t
// is fused into the pass that rescores the active region for block t+1.
#include <climits>

#include "pwp_internal.cuh"

namespace pwp {

// ------------------------------------------------------------------ setup kernels

__global__ void init_ctl_kernel(Ctl* ctl, long long zstar, pwp_stats* st, long long target) {
  ctl->zstar = zstar;
  ctl->pruned = 0;
  ctl->mode = 0;
  st->status = PWP_OK;
  st->status_site = 0;
  st->pruned = 0;
  st->target = target;
  st->lambda = 0.f;
  st->shortfall = 0;
  st->reread_blocks = 0;
  st->tie_blocks = 0;
}

__global__ void convert_w_kernel(const void* __restrict__ W, int wtype, float* __restrict__ Wout,
                                 long long N) {
  long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  long long stride = (long long)gridDim.x * blockDim.x;
  if (wtype == PWP_FP32) {
    const float* w = (const float*)W;
    for (; i < N; i += stride) Wout[i] = w[i];
  } else {
    const uint16_t* w = (const uint16_t*)W;
    for (; i < N; i += stride) Wout[i] = __uint_as_float(((unsigned int)w[i]) << 16);
  }
}

// ||X_q|| = sqrt(G_qq) for the Wanda score, U_qq for the OBS score.
__global__ void prep_diag_kernel(const float* __restrict__ H, int b, const float* __restrict__ g_diag,
                                 float* __restrict__ xnorm, float* __restrict__ udiag) {
  int q = blockIdx.x * blockDim.x + threadIdx.x;
  if (q < b) {
    xnorm[q] = sqrtf(g_diag[q]);
    udiag[q] = H[(long long)q * b + q];
  }
}

// Per block t: Hb = U_JJ^T U_JJ (B x B) and UJt[q][p] = U[j+p][j+q] (U_JJ transposed).
__global__ void __launch_bounds__(256) block_mats_kernel(const float* __restrict__ H, int b, int B,
                                                         float* __restrict__ Hb_all,
                                                         float* __restrict__ UJt_all,
                                                         const pwp_stats* st) {
  extern __shared__ float Us[];  // [B][B+1]
  if (failed(st)) return;
  const int t = blockIdx.x;
  const int j = t * B, nJ = min(B, b - j);
  const int ld = B + 1;
  for (int idx = threadIdx.x; idx < B * B; idx += blockDim.x) {
    int p = idx / B, q = idx % B;
    Us[p * ld + q] = (p < nJ && q < nJ && p <= q) ? H[(long long)(j + p) * b + j + q] : 0.f;
  }
  __syncthreads();
  float* Hb = Hb_all + (size_t)t * B * B;
  float* UJt = UJt_all + (size_t)t * B * B;
  for (int idx = threadIdx.x; idx < B * B; idx += blockDim.x) {
    int a = idx / B, c = idx % B;
    float s = 0.f;
    int lim = min(a, c);
    for (int p = 0; p <= lim; ++p) s = fmaf(Us[p * ld + a], Us[p * ld + c], s);
    Hb[idx] = s;
    UJt[idx] = Us[c * ld + a];  // UJt[a][c] = U[j+c][j+a]
  }
}

// ------------------------------------------------------------------ stream (update + score + histogram)

enum ScoreKind { kNoScore = 0, kWanda = 1, kObs = 2 };

template <int SCORE>
__device__ __forceinline__ unsigned int key_of(float w, float p) {
  return SCORE == kWanda ? score_key(wanda_score(w, p)) : score_key(obs_score(w, p));
}

// W[:, j:b] -= Zp[:, 0:Bp] * U[jp:jp+Bp, j:b]; then (SCORE != 0) histogram of the key
// bits [30:16] of every updated entry in columns [j, hist_end).
// Tiles of 64 rows x 128 columns, persistent grid-stride loop.
template <int SCORE>
__global__ void __launch_bounds__(256) stream_kernel(float* __restrict__ W, int c, int b, int j,
                                                     const float* __restrict__ Zp, int Bp, int ldz,
                                                     const float* __restrict__ H, int jp,
                                                     const float* __restrict__ sc, int hist_end,
                                                     unsigned int* __restrict__ hist1,
                                                     const pwp_stats* st) {
  extern __shared__ unsigned int shist[];  // kHist1Bins when SCORE != 0
  __shared__ float Zs[64][33];
  __shared__ float Us[32][128];
  if (failed(st)) return;
  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;
  if (SCORE != kNoScore)
    for (int i = tid; i < kHist1Bins; i += blockDim.x) shist[i] = 0u;
  const int ncols = b - j;
  const int tiles_c = (ncols + 127) / 128, tiles_r = (c + 63) / 64;
  const long long ntiles = (long long)tiles_c * tiles_r;
  __syncthreads();
  for (long long tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
    const int r0 = (int)(tile / tiles_c) * 64;
    const int c0 = j + (int)(tile % tiles_c) * 128;
    float acc[4][8];
#pragma unroll
    for (int x = 0; x < 4; ++x)
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        int r = r0 + ty + 16 * x, q = c0 + tx + 16 * e;
        acc[x][e] = (r < c && q < b) ? W[(long long)r * b + q] : 0.f;
      }
    for (int k0 = 0; k0 < Bp; k0 += 32) {
      for (int idx = tid; idx < 64 * 32; idx += 256) {
        int rr = idx >> 5, kk = idx & 31;
        int r = r0 + rr, k = k0 + kk;
        Zs[rr][kk] = (r < c && k < Bp) ? Zp[(long long)r * ldz + k] : 0.f;
      }
      for (int idx = tid; idx < 32 * 128; idx += 256) {
        int kk = idx >> 7, cc = idx & 127;
        int k = k0 + kk, q = c0 + cc;
        Us[kk][cc] = (k < Bp && q < b) ? H[(long long)(jp + k) * b + q] : 0.f;
      }
      __syncthreads();
#pragma unroll 4
      for (int kk = 0; kk < 32; ++kk) {
        float zv[4], uv[8];
#pragma unroll
        for (int x = 0; x < 4; ++x) zv[x] = Zs[ty + 16 * x][kk];
#pragma unroll
        for (int e = 0; e < 8; ++e) uv[e] = Us[kk][tx + 16 * e];
#pragma unroll
        for (int x = 0; x < 4; ++x)
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[x][e] = fmaf(-zv[x], uv[e], acc[x][e]);
      }
      __syncthreads();
    }
#pragma unroll
    for (int x = 0; x < 4; ++x) {
      int r = r0 + ty + 16 * x;
      if (r >= c) continue;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        int q = c0 + tx + 16 * e;
        if (q >= b) continue;
        if (Bp > 0) W[(long long)r * b + q] = acc[x][e];
        if (SCORE != kNoScore && q < hist_end) {
          unsigned int key = key_of<SCORE>(acc[x][e], __ldg(sc + q));
          atomicAdd(&shist[key >> 16], 1u);
        }
      }
    }
  }
  if (SCORE != kNoScore) {
    __syncthreads();
    for (int i = tid; i < kHist1Bins; i += blockDim.x) {
      unsigned int v = shist[i];
      if (v) atomicAdd(&hist1[i], v);
    }
  }
}

// ------------------------------------------------------------------ exact selection

__device__ __forceinline__ long long block_excl_scan(long long v, long long* sh, long long* total) {
  // 1024 threads; sh has >= 32 entries
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  long long x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    long long y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) sh[warp] = x;
  __syncthreads();
  if (warp == 0) {
    long long w = (lane < (blockDim.x >> 5)) ? sh[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      long long y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    sh[lane] = w;
  }
  __syncthreads();
  long long before_warp = warp ? sh[warp - 1] : 0;
  *total = sh[(blockDim.x >> 5) - 1];
  long long incl = before_warp + x;
  __syncthreads();
  return incl - v;
}

// Level 1: from the bits-[30:16] histogram find the bin holding the take-th smallest key.
// take = min(r, region) with r = zstar - pruned (global budget) or the block quota.
__global__ void __launch_bounds__(1024) pick1_kernel(Ctl* ctl, unsigned int* __restrict__ hist1,
                                                     unsigned int* __restrict__ hist2,
                                                     long long region_n, int global_budget,
                                                     long long quota, pwp_stats* st) {
  __shared__ long long sh[32];
  __shared__ long long s_take;
  __shared__ int s_found;
  if (failed(st)) return;
  const int tid = threadIdx.x;
  if (tid == 0) {
    long long r = global_budget ? ctl->zstar - ctl->pruned : quota;
    long long take = r < region_n ? r : region_n;
    if (take < r) st->shortfall = 1;
    if (take < 0) take = 0;
    ctl->take = take;
    s_take = take;
    s_found = 0;
    ctl->mode = take > 0 ? 1 : 0;
  }
  __syncthreads();
  const long long take = s_take;
  constexpr int PER = kHist1Bins / 1024;  // 32 bins per thread
  long long mine = 0;
  if (take > 0) {
    for (int i = 0; i < PER; ++i) mine += hist1[tid * PER + i];
  }
  long long total;
  long long before = block_excl_scan(mine, sh, &total);
  if (take > 0 && before < take && take <= before + mine) {
    long long cum = before;
    for (int i = 0; i < PER; ++i) {
      unsigned int h = hist1[tid * PER + i];
      if (take <= cum + h) {
        ctl->b1 = (unsigned int)(tid * PER + i);
        ctl->r1 = (unsigned int)(take - cum);
        ctl->count_less = cum;
        s_found = 1;
        break;
      }
      cum += h;
    }
  }
  __syncthreads();
  if (tid == 0 && take > 0 && !s_found) set_error(st, PWP_EBUDGET, kSitePick);
  for (int i = tid; i < kHist1Bins; i += blockDim.x) hist1[i] = 0u;
  for (int i = tid; i < kHist2Bins; i += blockDim.x) hist2[i] = 0u;
}

// Level 2 input: histogram of key bits [15:0] for entries whose top bits equal b1.
template <int SCORE>
__global__ void __launch_bounds__(256) refine_kernel(const float* __restrict__ W, int c, int b, int q0,
                                                     int q1, const float* __restrict__ sc,
                                                     const Ctl* __restrict__ ctl,
                                                     unsigned int* __restrict__ hist2,
                                                     const pwp_stats* st) {
  if (failed(st) || ctl->mode == 0) return;
  const unsigned int b1 = ctl->b1;
  const int w = q1 - q0;
  const long long N = (long long)c * w;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < N;
       i += (long long)gridDim.x * blockDim.x) {
    int r = (int)(i / w), q = q0 + (int)(i % w);
    unsigned int key = key_of<SCORE>(W[(long long)r * b + q], __ldg(sc + q));
    if ((key >> 16) == b1) atomicAdd(&hist2[key & 0xffffu], 1u);
  }
}

// Level 2: exact threshold key T, the number of entries below it, and -- when only
// some of the entries tied at T may be taken -- the column-major position inside the
// block [j, j1) of the last tied entry taken.  Ties are taken in (column, row) order.
template <int SCORE>
__global__ void __launch_bounds__(1024) pick2_kernel(Ctl* ctl, const unsigned int* __restrict__ hist2,
                                                     const float* __restrict__ W, int c, int b, int j,
                                                     int j1, const float* __restrict__ sc,
                                                     pwp_stats* st) {
  __shared__ long long sh[32];
  __shared__ int s_lo;
  __shared__ long long s_before;
  __shared__ unsigned int colcnt[kMaxBlock];
  __shared__ int s_qstar;
  __shared__ long long s_need;
  if (failed(st) || ctl->mode == 0) return;
  const int tid = threadIdx.x;
  const long long r1 = ctl->r1;
  constexpr int PER = kHist2Bins / 1024;  // 64
  long long mine = 0;
  for (int i = 0; i < PER; ++i) mine += hist2[tid * PER + i];
  if (tid == 0) s_lo = -1;
  long long total;
  long long before = block_excl_scan(mine, sh, &total);
  if (before < r1 && r1 <= before + mine) {
    long long cum = before;
    for (int i = 0; i < PER; ++i) {
      unsigned int h = hist2[tid * PER + i];
      if (r1 <= cum + h) {
        s_lo = tid * PER + i;
        s_before = cum;
        break;
      }
      cum += h;
    }
  }
  __syncthreads();
  if (s_lo < 0) {
    if (tid == 0) set_error(st, PWP_EBUDGET, kSitePick);
    return;
  }
  const unsigned int T = (ctl->b1 << 16) | (unsigned int)s_lo;
  const long long ties = hist2[s_lo];
  const long long count_less = ctl->count_less + s_before;
  const long long m = ctl->take - count_less;  // 1 <= m <= ties
  if (tid == 0) {
    ctl->T = T;
    ctl->ties = ties;
    ctl->m = m;
    ctl->count_less = count_less;
    ctl->pstar = LLONG_MAX;
    if (ties > 1) st->tie_blocks += 1;
  }
  if (m >= ties) return;  // every tied entry is taken
  // Some but not all ties are taken: count ties per block column (rows coalesced).
  const int nJ = j1 - j;
  for (int i = tid; i < kMaxBlock; i += blockDim.x) colcnt[i] = 0u;
  __syncthreads();
  const int warp = tid >> 5, lane = tid & 31;
  for (int r = warp; r < c; r += 32) {
    for (int qq = lane; qq < nJ; qq += 32) {
      unsigned int key = key_of<SCORE>(W[(long long)r * b + j + qq], __ldg(sc + j + qq));
      if (key == T) atomicAdd(&colcnt[qq], 1u);
    }
  }
  __syncthreads();
  if (tid == 0) {
    long long cum = 0;
    int qstar = -1;
    for (int qq = 0; qq < nJ; ++qq) {
      if (cum + colcnt[qq] >= m) { qstar = qq; break; }
      cum += colcnt[qq];
    }
    s_qstar = qstar;
    s_need = m - cum;  // 1-based rank of the last taken tie inside column qstar
  }
  __syncthreads();
  if (s_qstar < 0) return;  // fewer than m ties inside the block: all of them are taken
  // find the row of the s_need-th tie (row order) in column qstar
  const int q = j + s_qstar;
  const int per = (c + 1023) / 1024;
  long long cnt = 0;
  for (int i = 0; i < per; ++i) {
    int r = tid * per + i;
    if (r < c && key_of<SCORE>(W[(long long)r * b + q], __ldg(sc + q)) == T) ++cnt;
  }
  long long tot;
  long long bef = block_excl_scan(cnt, sh, &tot);
  const long long need = s_need;
  if (bef < need && need <= bef + cnt) {
    long long k = bef;
    for (int i = 0; i < per; ++i) {
      int r = tid * per + i;
      if (r < c && key_of<SCORE>(W[(long long)r * b + q], __ldg(sc + q)) == T) {
        if (++k == need) {
          ctl->pstar = (long long)s_qstar * c + r;
          break;
        }
      }
    }
  }
}

// ------------------------------------------------------------------ per-row work

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Selection flag of one entry of the block.  Unstructured: key < T, or key == T and its
// column-major position in the block is at or before pstar.  N:M: rank inside the
// group of m lanes by (key, column) below m - n.  All lanes of the warp must call it.
template <int SCORE, bool NM>
__device__ __forceinline__ bool selected(unsigned int key, bool valid, int qq, int k, int c,
                                         const Ctl& ctl, int nm_n, int nm_m) {
  if (NM) {
    const int lane = threadIdx.x & 31;
    const int base = lane & ~(nm_m - 1);
    int rank = 0;
    for (int o = 0; o < nm_m; ++o) {
      unsigned int ko = __shfl_sync(0xffffffffu, key, base + o);
      int lo = base + o;
      rank += (ko < key) || (ko == key && lo < lane);
    }
    return valid && rank < nm_m - nm_n;
  }
  if (!valid || ctl.mode == 0) return false;
  if (key < ctl.T) return true;
  if (key == ctl.T) return (long long)qq * c + k <= ctl.pstar;
  return false;
}

// Thanos per-row joint solve, one warp per row.
// smem per warp: Qidx[B] ints, vec[B] floats, L[B(B+1)/2] floats (packed lower).
template <bool NM>
__global__ void __launch_bounds__(128) thanos_solve_kernel(float* __restrict__ W, int c, int b, int j,
                                                           int B, const float* __restrict__ Hb,
                                                           const float* __restrict__ UJt,
                                                           const float* __restrict__ xnorm,
                                                           const Ctl* __restrict__ ctlp,
                                                           uint8_t* __restrict__ mask,
                                                           float* __restrict__ Zp, int nm_n, int nm_m,
                                                           Ctl* __restrict__ ctl_out, pwp_stats* st) {
  extern __shared__ float smem[];
  if (failed(st)) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int per_warp = 2 * B + B * (B + 1) / 2;
  int* Qidx = (int*)(smem + warp * per_warp);
  float* vec = smem + warp * per_warp + B;
  float* L = vec + B;
  const Ctl ctl = *ctlp;
  const int nJ = min(B, b - j);
  const int k = blockIdx.x * (blockDim.x >> 5) + warp;
  if (k >= c) return;
  constexpr int MAXI = kMaxBlock / 32;
  float w[MAXI];
  bool sel[MAXI];
  float* wrow = W + (long long)k * b + j;
  int s = 0;
#pragma unroll
  for (int i = 0; i < MAXI; ++i) {
    const int qq = lane + 32 * i;
    const bool valid = qq < nJ;
    w[i] = valid ? wrow[qq] : 0.f;
    unsigned int key = valid ? key_of<kWanda>(w[i], __ldg(xnorm + j + qq)) : 0xffffffffu;
    sel[i] = (32 * i < nJ) ? selected<kWanda, NM>(key, valid, qq, k, c, ctl, nm_n, nm_m) : false;
    unsigned int bal = __ballot_sync(0xffffffffu, sel[i]);
    if (sel[i]) {
      int pos = s + __popc(bal & ((1u << lane) - 1u));
      Qidx[pos] = qq;
      vec[pos] = w[i];
    }
    s += __popc(bal);
  }
  __syncwarp();
  bool ok = true;
  if (s > 0) {
    // R-hat = Hb[Q, Q], lower triangle packed by rows
    const int npk = s * (s + 1) / 2;
    for (int idx = lane; idx < npk; idx += 32) {
      int a = (int)((sqrtf(8.f * idx + 1.f) - 1.f) * 0.5f);
      while ((a + 1) * (a + 2) / 2 <= idx) ++a;
      while (a * (a + 1) / 2 > idx) --a;
      int cc = idx - a * (a + 1) / 2;
      L[idx] = Hb[(size_t)Qidx[a] * B + Qidx[cc]];
    }
    __syncwarp();
    // Cholesky, left-looking by columns
    for (int jj = 0; jj < s && ok; ++jj) {
      float* rj = L + jj * (jj + 1) / 2;
      float part = 0.f;
      for (int t = lane; t < jj; t += 32) part = fmaf(rj[t], rj[t], part);
      float d = rj[jj] - warp_sum(part);
      if (!(d > 0.f)) { ok = false; break; }
      float ljj = sqrtf(d);
      float inv = 1.f / ljj;
      __syncwarp();
      if (lane == 0) rj[jj] = ljj;
      for (int a = jj + 1 + lane; a < s; a += 32) {
        float* ra = L + a * (a + 1) / 2;
        float acc = ra[jj];
        for (int t = 0; t < jj; ++t) acc = fmaf(-ra[t], rj[t], acc);
        ra[jj] = acc * inv;
      }
      __syncwarp();
    }
    if (ok) {
      // forward: L y = u
      for (int a = 0; a < s; ++a) {
        const float* ra = L + a * (a + 1) / 2;
        float part = 0.f;
        for (int t = lane; t < a; t += 32) part = fmaf(ra[t], vec[t], part);
        float y = (vec[a] - warp_sum(part)) / ra[a];
        __syncwarp();
        if (lane == 0) vec[a] = y;
        __syncwarp();
      }
      // backward: L^T z = y
      for (int a = s - 1; a >= 0; --a) {
        float part = 0.f;
        for (int t = a + 1 + lane; t < s; t += 32) part = fmaf(L[t * (t + 1) / 2 + a], vec[t], part);
        float z = (vec[a] - warp_sum(part)) / L[a * (a + 1) / 2 + a];
        __syncwarp();
        if (lane == 0) vec[a] = z;
        __syncwarp();
      }
    } else if (lane == 0) {
      set_error(st, PWP_ENOTSPD, kSiteSolve);
    }
  }
  // in-block update, exact zeros, mask, Z' = U_JJ z
  uint8_t* mrow = mask + (long long)k * b + j;
  float* zrow = Zp + (long long)k * B;
#pragma unroll
  for (int i = 0; i < MAXI; ++i) {
    const int qq = lane + 32 * i;
    if (qq < nJ) {
      float d = 0.f, zq = 0.f;
      for (int a = 0; a < s; ++a) {
        float za = vec[a];
        d = fmaf(za, Hb[(size_t)Qidx[a] * B + qq], d);
        zq = fmaf(za, UJt[(size_t)Qidx[a] * B + qq], zq);
      }
      float v = sel[i] ? 0.f : w[i] - d;
      wrow[qq] = v;
      mrow[qq] = sel[i] ? 1 : 0;
      zrow[qq] = (s > 0 && ok) ? zq : 0.f;
    } else if (qq < B) {
      zrow[qq] = 0.f;
    }
  }
  if (lane == 0 && s > 0) atomicAdd((unsigned long long*)&ctl_out->pruned, (unsigned long long)s);
}

// SparseGPT in-block column sweep, one warp per row: for each block column q in order,
// e = W_q / U_qq on a selected entry (0 otherwise), W[q+1:j1] -= e U[q, q+1:j1], W_q = 0.
// E (the e values) feeds the trailing update like Thanos's Z'.
template <bool NM>
__global__ void __launch_bounds__(256) sparsegpt_solve_kernel(float* __restrict__ W, int c, int b, int j,
                                                              int B, const float* __restrict__ H,
                                                              const float* __restrict__ udiag,
                                                              const Ctl* __restrict__ ctlp,
                                                              uint8_t* __restrict__ mask,
                                                              float* __restrict__ Zp, int nm_n, int nm_m,
                                                              Ctl* __restrict__ ctl_out, pwp_stats* st) {
  if (failed(st)) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int k = blockIdx.x * (blockDim.x >> 5) + warp;
  if (k >= c) return;
  const Ctl ctl = *ctlp;
  const int nJ = min(B, b - j);
  constexpr int MAXI = kMaxBlock / 32;
  float w[MAXI], e[MAXI];
  bool sel[MAXI];
  float* wrow = W + (long long)k * b + j;
  int s = 0;
#pragma unroll
  for (int i = 0; i < MAXI; ++i) {
    const int qq = lane + 32 * i;
    const bool valid = qq < nJ;
    w[i] = valid ? wrow[qq] : 0.f;
    e[i] = 0.f;
    unsigned int key = valid ? key_of<kObs>(w[i], __ldg(udiag + j + qq)) : 0xffffffffu;
    sel[i] = (32 * i < nJ) ? selected<kObs, NM>(key, valid, qq, k, c, ctl, nm_n, nm_m) : false;
    s += __popc(__ballot_sync(0xffffffffu, sel[i]));
  }
  for (int qq = 0; qq < nJ; ++qq) {
    const int owner = qq & 31, slot = qq >> 5;
    float wq = 0.f;
    bool sq = false;
#pragma unroll
    for (int i = 0; i < MAXI; ++i)
      if (i == slot) { wq = w[i]; sq = sel[i]; }
    wq = __shfl_sync(0xffffffffu, wq, owner);
    sq = __shfl_sync(0xffffffffu, sq, owner);
    if (!sq) continue;
    const float ev = wq / __ldg(udiag + j + qq);
    const float* urow = H + (long long)(j + qq) * b + j;
#pragma unroll
    for (int i = 0; i < MAXI; ++i) {
      const int p = lane + 32 * i;
      if (p > qq && p < nJ) w[i] = fmaf(-ev, urow[p], w[i]);
      if (p == qq) { w[i] = 0.f; e[i] = ev; }
    }
  }
  uint8_t* mrow = mask + (long long)k * b + j;
  float* zrow = Zp + (long long)k * B;
#pragma unroll
  for (int i = 0; i < MAXI; ++i) {
    const int qq = lane + 32 * i;
    if (qq < nJ) {
      wrow[qq] = sel[i] ? 0.f : w[i];
      mrow[qq] = sel[i] ? 1 : 0;
      zrow[qq] = e[i];
    } else if (qq < B) {
      zrow[qq] = 0.f;
    }
  }
  if (lane == 0 && s > 0) atomicAdd((unsigned long long*)&ctl_out->pruned, (unsigned long long)s);
}

__global__ void finalize_kernel(const Ctl* ctl, pwp_stats* st, int check_budget) {
  st->pruned = ctl->pruned;
  if (st->status == PWP_OK && check_budget && ctl->pruned != ctl->zstar)
    set_error(st, PWP_EBUDGET, kSiteFinal);
}

// ------------------------------------------------------------------ host driver

struct PruneBuffers {
  Ctl* ctl;
  unsigned int* hist1;
  unsigned int* hist2;
  float* g_diag;
  float* xnorm;
  float* udiag;
  float* Zp;
  float* Hb;
  float* UJt;
  void* fws;
  size_t fws_bytes;
};

static size_t align_up(size_t x) { return (x + 255) & ~(size_t)255; }

size_t prune_ws_layout(int c, int b, int B, PruneBuffers* pb, char* base) {
  const int nblk = (b + B - 1) / B;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off += align_up(bytes);
    return base ? (void*)(base + o) : nullptr;
  };
  PruneBuffers t;
  t.ctl = (Ctl*)take(sizeof(Ctl));
  t.hist1 = (unsigned int*)take(sizeof(unsigned int) * kHist1Bins);
  t.hist2 = (unsigned int*)take(sizeof(unsigned int) * kHist2Bins);
  t.g_diag = (float*)take(sizeof(float) * b);
  t.xnorm = (float*)take(sizeof(float) * b);
  t.udiag = (float*)take(sizeof(float) * b);
  t.Zp = (float*)take(sizeof(float) * (size_t)c * B);
  t.Hb = (float*)take(sizeof(float) * (size_t)nblk * B * B);
  t.UJt = (float*)take(sizeof(float) * (size_t)nblk * B * B);
  t.fws_bytes = factor_ws_bytes(b);
  t.fws = take(t.fws_bytes);
  if (pb) *pb = t;
  return off;
}

static int g_stream_grid = 0;

cudaError_t launch_prune(const pwp_config* cfg, const void* W, int wtype, int c, int b, float* H,
                         float* Wout, uint8_t* mask, void* ws, pwp_stats* st, cudaStream_t s) {
  PruneBuffers pb;
  const int B = cfg->block;
  prune_ws_layout(c, b, B, &pb, (char*)ws);
  const bool thanos = cfg->method == PWP_THANOS;
  const bool nm = cfg->pattern == PWP_NM;
  const long long N = (long long)c * b;
  const long long zstar = (long long)((double)cfg->sparsity * (double)N);
  long long target = 0;
  const int nblk = (b + B - 1) / B;
  if (nm) {
    target = N / cfg->nm_m * (cfg->nm_m - cfg->nm_n);
  } else if (thanos) {
    target = zstar;
  } else {
    for (int t = 0; t < nblk; ++t) {
      int nJ = min(B, b - t * B);
      target += (long long)((double)cfg->sparsity * (double)c * (double)nJ);
    }
  }
  static bool attrs = false;
  if (!attrs) {
    cudaFuncSetAttribute(stream_kernel<kWanda>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         kHist1Bins * 4);
    cudaFuncSetAttribute(stream_kernel<kObs>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         kHist1Bins * 4);
    const int solve_smem = 4 * (2 * kMaxBlock + kMaxBlock * (kMaxBlock + 1) / 2) * 4;
    cudaFuncSetAttribute(thanos_solve_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         solve_smem);
    cudaFuncSetAttribute(thanos_solve_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         solve_smem);
    cudaFuncSetAttribute(block_mats_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         kMaxBlock * (kMaxBlock + 1) * 4);
    int dev = 0, nsm = kNumSM;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
    g_stream_grid = nsm;
    attrs = true;
  }
  long long nl = 0;
  init_ctl_kernel<<<1, 1, 0, s>>>(pb.ctl, zstar, st, target);
  cudaMemsetAsync(pb.hist1, 0, sizeof(unsigned int) * kHist1Bins, s);
  convert_w_kernel<<<4 * g_stream_grid, 256, 0, s>>>(W, wtype, Wout, N);
  nl += 2;
  prof_begin(kKFactor, s);
  cudaError_t e = launch_damp_factor(H, b, cfg->damp, pb.g_diag, pb.fws, pb.fws_bytes, st, s);
  prof_end(kKFactor, s);
  if (e != cudaSuccess) return e;
  prep_diag_kernel<<<(b + 255) / 256, 256, 0, s>>>(H, b, pb.g_diag, pb.xnorm, pb.udiag);
  block_mats_kernel<<<nblk, 256, B * (B + 1) * 4, s>>>(H, b, B, pb.Hb, pb.UJt, st);
  nl += 2;

  const int solve_smem = 4 * (2 * B + B * (B + 1) / 2) * 4;
  for (int t = 0; t < nblk; ++t) {
    const int j = t * B, j1 = min(b, j + B);
    const int jp = (t - 1) * B, Bp = t > 0 ? (j - jp) : 0;
    const float* Hb_t = pb.Hb + (size_t)t * B * B;
    const float* UJt_t = pb.UJt + (size_t)t * B * B;
    if (!nm && thanos) {
      // rescore the whole active region [j, b) while applying the previous block's update
      prof_begin(kKStream, s);
      stream_kernel<kWanda><<<g_stream_grid, 256, kHist1Bins * 4, s>>>(
          Wout, c, b, j, pb.Zp, Bp, B, H, jp, pb.xnorm, b, pb.hist1, st);
      prof_end(kKStream, s);
      prof_begin(kKSelect, s);
      pick1_kernel<<<1, 1024, 0, s>>>(pb.ctl, pb.hist1, pb.hist2, (long long)c * (b - j), 1, 0, st);
      refine_kernel<kWanda><<<4 * g_stream_grid, 256, 0, s>>>(Wout, c, b, j, b, pb.xnorm, pb.ctl,
                                                              pb.hist2, st);
      pick2_kernel<kWanda><<<1, 1024, 0, s>>>(pb.ctl, pb.hist2, Wout, c, b, j, j1, pb.xnorm, st);
      prof_end(kKSelect, s);
      nl += 4;
    } else if (!nm) {
      // SparseGPT: update the active region, score only the block
      prof_begin(kKStream, s);
      stream_kernel<kObs><<<g_stream_grid, 256, kHist1Bins * 4, s>>>(
          Wout, c, b, j, pb.Zp, Bp, B, H, jp, pb.udiag, j1, pb.hist1, st);
      prof_end(kKStream, s);
      prof_begin(kKSelect, s);
      long long quota = (long long)((double)cfg->sparsity * (double)c * (double)(j1 - j));
      pick1_kernel<<<1, 1024, 0, s>>>(pb.ctl, pb.hist1, pb.hist2, (long long)c * (j1 - j), 0, quota,
                                      st);
      refine_kernel<kObs><<<4 * g_stream_grid, 256, 0, s>>>(Wout, c, b, j, j1, pb.udiag, pb.ctl,
                                                            pb.hist2, st);
      pick2_kernel<kObs><<<1, 1024, 0, s>>>(pb.ctl, pb.hist2, Wout, c, b, j, j1, pb.udiag, st);
      prof_end(kKSelect, s);
      nl += 4;
    } else if (t > 0) {
      prof_begin(kKStream, s);
      stream_kernel<kNoScore><<<g_stream_grid, 256, 0, s>>>(Wout, c, b, j, pb.Zp, Bp, B, H, jp,
                                                            pb.xnorm, j, pb.hist1, st);
      prof_end(kKStream, s);
      nl += 1;
    }
    const int rows_per_cta = thanos ? 4 : 8;
    const int grid = (c + rows_per_cta - 1) / rows_per_cta;
    prof_begin(kKSolve, s);
    nl += 1;
    if (thanos) {
      if (nm)
        thanos_solve_kernel<true><<<grid, 128, solve_smem, s>>>(Wout, c, b, j, B, Hb_t, UJt_t,
                                                                pb.xnorm, pb.ctl, mask, pb.Zp,
                                                                cfg->nm_n, cfg->nm_m, pb.ctl, st);
      else
        thanos_solve_kernel<false><<<grid, 128, solve_smem, s>>>(Wout, c, b, j, B, Hb_t, UJt_t,
                                                                 pb.xnorm, pb.ctl, mask, pb.Zp,
                                                                 cfg->nm_n, cfg->nm_m, pb.ctl, st);
    } else {
      if (nm)
        sparsegpt_solve_kernel<true><<<grid, 256, 0, s>>>(Wout, c, b, j, B, H, pb.udiag, pb.ctl,
                                                          mask, pb.Zp, cfg->nm_n, cfg->nm_m,
                                                          pb.ctl, st);
      else
        sparsegpt_solve_kernel<false><<<grid, 256, 0, s>>>(Wout, c, b, j, B, H, pb.udiag, pb.ctl,
                                                           mask, pb.Zp, cfg->nm_n, cfg->nm_m,
                                                           pb.ctl, st);
    }
    prof_end(kKSolve, s);
  }
  finalize_kernel<<<1, 1, 0, s>>>(pb.ctl, st, (thanos && !nm) ? 1 : 0);
  count_launches(nl + 1);
  return cudaGetLastError();
}

}  // namespace pwp
