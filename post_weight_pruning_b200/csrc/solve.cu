// Per-row work of one column block: the mask, and the coefficients of the row's
// compensating update.
//
// Thanos ("Pruning LLMs with Thanos", section "Contribution one: solve a selected set
// directly"): for row k with selected set Q in block J, u = W[k, Q] and
// R-hat = K[Q, Q] with K = inv(H_d[A, A]); z = R-hat^-1 u and the row's update is
// delta_k = -z^T K[Q, A].  This kernel produces z (scattered into a B-wide row, zero
// outside Q); the stream kernel then applies W[:, A] -= Z K[J, A] for all rows at once,
// and sets W[k, Q] to exactly zero.  R-hat is gathered from the block's in-block inverse
// K[J, J] (B x B, row stride B).
//
// Both kernels store a row of Z as a TF32 head (rows 0..c-1 of Zs) and its exact fp32
// remainder (rows c..2c-1), the operand form of the tensor-core update.
//
// SparseGPT ("Weight Pruning in Large Language Models ...", section "SparseGPT"): the
// column-sequential sweep inside the block, e_q = W_q / U_qq on selected entries, whose
// in-block part is replayed here row by row to get e; the stream kernel applies
// W[:, A] -= E U[J, A].
#include "pwp_internal.cuh"

namespace pwp {
namespace {

// Packed lower-triangular storage with every row starting on a 16-byte boundary:
// row i holds entries 0..i and is padded to a multiple of 4 floats.
__host__ __device__ constexpr int poff(int i) {
  return 4 * (2 * (i >> 2) * ((i >> 2) + 1) + (i & 3) * ((i >> 2) + 1));
}

// Per warp: rows 0..kNS-1 of the packed factor, the u/y/z vector, the selected indices
// (reused for the pivots' reciprocals) and the staged 8x8 diagonal block, in shared
// memory; rows kNS..kCap-1 (only rows with more than kNS selections reach them) in a
// per-warp slot of global scratch, which stays in L2.
constexpr int kCap = kMaxBlock;      // largest selected set of a row
constexpr int kNS = kSolveNS;        // factor rows kept in shared memory
constexpr int kL = poff(kNS);
constexpr int kY = kCap + 8;
constexpr int kPerWarp = kL + kY + kCap + 64;        // floats: L, y, Qidx, D
constexpr int kGlobalPerWarp = poff(kCap) - poff(kNS);
constexpr int kSolveWarps = 8;
static_assert(kL % 4 == 0 && kY % 4 == 0 && kCap % 4 == 0, "16-byte aligned regions");

// Rows of the packed factor.  SMALL: every row lives in shared memory (s <= kNS), so all
// pointers stay shared-memory pointers; otherwise rows from kNS on are in global scratch.
template <bool SMALL>
struct Rows {
  float* L;   // shared, rows < kNS
  float* G;   // global, rows >= kNS
  __device__ __forceinline__ float* row(int i) const { return at(poff(i)); }
  // the row at packed offset off (row i + 1 starts 4 * (i / 4 + 1) floats after row i)
  __device__ __forceinline__ float* at(int off) const {
    if (SMALL) return L + off;
    return off < kL ? L + off : G + (off - kL);
  }
};

// Four bytes global -> shared without a register stop (completion: cp_async_wait_all)
__device__ __forceinline__ void cp_async4(float* sdst, const float* gsrc) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"((unsigned int)__cvta_generic_to_shared(sdst)),
               "l"(gsrc)
               : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

__device__ __forceinline__ float dot4(float4 a, float4 b, float acc) {
  acc = fmaf(-a.x, b.x, acc);
  acc = fmaf(-a.y, b.y, acc);
  acc = fmaf(-a.z, b.z, acc);
  return fmaf(-a.w, b.w, acc);
}

// acc[q][c] -= sum_{t < jp} row_q[t] * prow_c[t] for the NQ row slots of one pass.
template <int NQ>
__device__ __forceinline__ void panel_gemm(float (&acc)[2][8], const float* const (&rp)[2],
                                           const float* const (&pr)[8], int jp) {
#pragma unroll 1
  for (int t = 0; t < jp; t += 4) {
    float4 x[NQ];
#pragma unroll
    for (int q = 0; q < NQ; ++q) x[q] = *reinterpret_cast<const float4*>(rp[q] + t);
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const float4 p = *reinterpret_cast<const float4*>(pr[c] + t);
#pragma unroll
      for (int q = 0; q < NQ; ++q) acc[q][c] = dot4(x[q], p, acc[q][c]);
    }
  }
}

// Cholesky R-hat = L L^T of the s x s gathered matrix (its lower triangle in R on entry,
// L on return), left-looking over 8-column panels, with u carried as an extra row s so
// that the same sweep gives y = L^-1 u; then the back substitution L^T z = y.  On return
// y[0..s) = z.  Per panel [jp, jp+8) the rows i in [jp, s] go over the lanes, two rows per
// lane and pass (lane l: rows jp+l+64p and jp+l+64p+32): each takes the contributions of
// the columns before jp (float4 dot products with the eight panel rows, which every lane
// reads as broadcasts), then finishes its eight panel entries column by column.  In the
// first pass the panel's diagonal rows are slot 0 of lanes 0..7: at column c lane c's
// entries so far reach every lane by shuffles (each lane forms the pivot), so the diagonal block is
// factored and every row's panel entries solved in one sweep; a later pass reads the
// stored diagonal rows and reciprocal pivots instead.  A packed row i holds columns up to
// 4*(i/4)+3, so rows jp..jp+3 of a panel store only its first four columns; columns
// beyond i inside a row's padding are never read.  Reciprocal pivots go to idg for the
// back substitution.  Returns false on a non-positive pivot (uniform).
template <bool SMALL>
__device__ bool chol_solve(const Rows<SMALL> R, float* __restrict__ y, float* __restrict__ idg,
                           float* __restrict__ D, int s, int lane) {
  (void)D;
  int pan = 0;   // packed offset of row jp
  for (int jp = 0; jp < s; jp += 8) {
    const int pw = min(8, s - jp);
    // row jp + c starts c * (jp + 4) + 4 * max(c - 4, 0) floats after row jp
    const float* pr[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) pr[c] = R.at(pan + (c < pw ? c * (jp + 4) + (c > 4 ? 4 * (c - 4) : 0) : 0));
    for (int pass = 0; jp + 64 * pass <= s; ++pass) {
      const bool two = jp + 64 * pass + 32 <= s;   // uniform: some lane has a second row
      int ii[2];
      const float* rp[2];
      float acc[2][8];
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const int i = jp + lane + 64 * pass + 32 * q;
        ii[q] = i;
        float* r = i < s ? R.row(i) : y;           // row s is the u row; rows past it are idle
        rp[q] = r;
        const bool hi = i >= jp + 4 || i >= s;     // the row's storage holds panel columns jp+4..
        const float4 a = *reinterpret_cast<const float4*>(r + jp);
        float4 bq = make_float4(0.f, 0.f, 0.f, 0.f);
        if (hi) bq = *reinterpret_cast<const float4*>(r + jp + 4);
        acc[q][0] = a.x; acc[q][1] = a.y; acc[q][2] = a.z; acc[q][3] = a.w;
        acc[q][4] = bq.x; acc[q][5] = bq.y; acc[q][6] = bq.z; acc[q][7] = bq.w;
      }
      if (two) panel_gemm<2>(acc, rp, pr, jp);
      else panel_gemm<1>(acc, rp, pr, jp);
      float x[2][8];
      if (pass == 0) {
        bool ok = true;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          if (c < pw) {   // uniform
            float lc[8];
#pragma unroll
            for (int c2 = 0; c2 < c; ++c2) lc[c2] = __shfl_sync(0xffffffffu, x[0][c2], c);
            // the pivot, formed in every lane from lane c's entries (the same operations
            // in the same order as lane c's own v[0], so the same value)
            float d = __shfl_sync(0xffffffffu, acc[0][c], c);
#pragma unroll
            for (int c2 = 0; c2 < c; ++c2) d = fmaf(-lc[c2], lc[c2], d);
            float v[2];
#pragma unroll
            for (int q = 0; q < 2; ++q) {
              v[q] = acc[q][c];
#pragma unroll
              for (int c2 = 0; c2 < c; ++c2) v[q] = fmaf(-x[q][c2], lc[c2], v[q]);
            }
            ok = ok && (d > 0.f);
            const float il = rsqrtf(d);
            if (lane == 0) idg[jp + c] = il;
#pragma unroll
            for (int q = 0; q < 2; ++q) x[q][c] = v[q] * il;
          } else {
            x[0][c] = 0.f;
            x[1][c] = 0.f;
          }
        }
        if (!ok) return false;   // the same pivots in every lane
      } else {
        // the diagonal rows were stored by the first pass
        float il[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) il[c] = c < pw ? idg[jp + c] : 1.f;
#pragma unroll
        for (int q = 0; q < 2; ++q) {
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            float v = acc[q][c];
#pragma unroll
            for (int c2 = 0; c2 < c; ++c2) v = fmaf(-x[q][c2], pr[c][jp + c2], v);
            x[q][c] = v * il[c];
          }
        }
      }
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        if (q == 1 && !two) break;
        const int i = ii[q];
        if (i > s) continue;
        float* r = const_cast<float*>(rp[q]);
        *reinterpret_cast<float4*>(r + jp) = make_float4(x[q][0], x[q][1], x[q][2], x[q][3]);
        if (i >= jp + 4 || i >= s)
          *reinterpret_cast<float4*>(r + jp + 4) = make_float4(x[q][4], x[q][5], x[q][6], x[q][7]);
      }
      __syncwarp();   // a later pass reads the stored diagonal rows
    }
    pan += 8 * jp + 48;   // rows jp .. jp+7: 4 * (jp/4 + 1) floats each, +4 for the second four
  }
  // back substitution L^T z = y from the bottom, one unknown at a time with y held in
  // registers (lane l: y[l + 32q]): the owner of unknown i forms z_i = y_i / L_ii and
  // broadcasts it, and every lane drops z_i L[i][t] from its y_t, t < i (row i of the
  // packed factor, read along its length)
  constexpr int CH = SMALL ? (kNS + 31) / 32 : (kCap + 31) / 32;
  float yv[CH], dv[CH];
#pragma unroll
  for (int q = 0; q < CH; ++q) {
    const int t = lane + 32 * q;
    yv[q] = t < s ? y[t] : 0.f;
    dv[q] = t < s ? idg[t] : 0.f;
  }
  int off = poff(s - 1);
#pragma unroll
  for (int qc = CH - 1; qc >= 0; --qc) {
    if (32 * qc >= s) continue;
#pragma unroll 4
    for (int i = min(s, 32 * qc + 32) - 1; i >= 32 * qc; --i) {
      const int src = i & 31;
      const float zi = __shfl_sync(0xffffffffu, yv[qc] * dv[qc], src);
      const float* Li = R.at(off);
      off -= 4 * ((i - 1) >> 2) + 4;   // row i - 1 (unused past row 0)
#pragma unroll
      for (int q = 0; q <= qc; ++q) {
        const int t = lane + 32 * q;
        if (q < qc || t < i) yv[q] = fmaf(-Li[t], zi, yv[q]);
      }
      if (lane == src) yv[qc] = zi;
    }
  }
  __syncwarp();
#pragma unroll
  for (int q = 0; q < CH; ++q) {
    const int t = lane + 32 * q;
    if (t < s) y[t] = yv[q];
  }
  __syncwarp();
  return true;
}

// R-hat = K[Q, Q], lower triangle, into the packed rows: entry (a, cc), cc <= a, is
// K[q_a, q_cc], copied straight from K's row q_a (lane l takes columns q_l, q_{l+32}, ...;
// one copy instruction stays inside one 512-byte row) by asynchronous copies into shared
// memory, all of them in flight before one wait (rows past the shared ones, on the
// general path, go through registers).
template <bool SMALL>
__device__ void gather_rhat(const Rows<SMALL> R, const float* __restrict__ Kt, const int* __restrict__ Qidx, int s,
                            int B, int lane) {
  constexpr int CH = SMALL ? (kNS + 31) / 32 : (kCap + 31) / 32;
  int qv[CH];
#pragma unroll
  for (int ch = 0; ch < CH; ++ch) qv[ch] = (lane + 32 * ch < s) ? Qidx[lane + 32 * ch] : 0;
  int off = 0;
#pragma unroll 4
  for (int a = 0; a < s; ++a) {
    const int hc = a >> 5;   // uniform
    int qsrc = qv[0];
#pragma unroll
    for (int ch = 1; ch < CH; ++ch)
      if (hc == ch) qsrc = qv[ch];
    const int qa = __shfl_sync(0xffffffffu, qsrc, a & 31);
    const float* krow = Kt + (size_t)qa * B;
    float* row = R.at(off);
    const bool shared_row = SMALL || off < kL;
#pragma unroll
    for (int ch = 0; ch < CH; ++ch) {
      if (ch <= hc && lane + 32 * ch <= a) {
        if (shared_row) cp_async4(row + lane + 32 * ch, krow + qv[ch]);
        else row[lane + 32 * ch] = __ldg(krow + qv[ch]);
      }
    }
    off += 4 * ((a >> 2) + 1);
  }
  cp_async_wait_all();
  __syncwarp();
}

// One warp per row over a persistent grid (each warp keeps one shared-memory slab and one
// global scratch slot).  A row whose selected set fits the shared rows takes the
// shared-memory-only path; a larger one (rows past kNS in the warp's global slot) the
// general path.
template <bool NM>
__global__ void __launch_bounds__(kSolveWarps * 32, 2) thanos_solve_kernel(const float* __restrict__ W, int c,
                                                                          int b, int j, int B,
                                                                          const float* __restrict__ Kt,
                                                                          const float* __restrict__ xnorm,
                                                                          Ctl* __restrict__ ctlp, Level2 l2,
                                                                          uint8_t* __restrict__ mask,
                                                                          float* __restrict__ Zs, int nm_n, int nm_m,
                                                                          float* __restrict__ gscratch,
                                                                          pwp_stats* st) {
  pdl_enter();
  extern __shared__ __align__(16) float smem[];
  if (warp_failed(st)) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nwarps = blockDim.x >> 5;
  const int slot = blockIdx.x * nwarps + warp;
  float* L = smem + warp * kPerWarp;
  float* y = L + kL;
  int* Qidx = reinterpret_cast<int*>(y + kY);
  float* D = reinterpret_cast<float*>(Qidx + kCap);
  float* G = gscratch ? gscratch + (size_t)slot * kGlobalPerWarp : nullptr;
  const Ctl ctl = *ctlp;
  clear_used_level2(ctl, l2, blockIdx.x * blockDim.x + threadIdx.x, gridDim.x * blockDim.x);
  const int nJ = min(B, b - j);
  constexpr int MAXI = kMaxBlock / 32;
  // the size of row k's selected set (nothing written)
  auto count_selected = [&](int k) -> int {
    const float* wrow = W + (long long)k * b + j;
    int s = 0;
#pragma unroll
    for (int i = 0; i < MAXI; ++i) {
      const int qq = lane + 32 * i;
      const bool valid = qq < nJ;
      const float w = valid ? wrow[qq] : 0.f;
      const unsigned int key = valid ? key_of<kWanda>(w, __ldg(xnorm + j + qq)) : 0xffffffffu;
      const bool sel = (32 * i < nJ) ? selected<NM>(key, valid, qq, k, c, ctl, nm_n, nm_m) : false;
      s += __popc(__ballot_sync(0xffffffffu, sel));
    }
    return s;
  };
  // row k's whole work; with small_only a row whose set exceeds kNS is left (after its mask
  // bytes, which its slice's warp writes identically) to that warp
  auto solve_row = [&](int k, bool small_only) {
    const float* wrow = W + (long long)k * b + j;
    uint8_t* mrow = mask + (long long)k * b + j;
    // the selection: mask bytes, the selected indices and u = W[k, Q]; the warp keeps only
    // the count (the positions are recounted from the mask bytes for the output)
    int s = 0;
#pragma unroll
    for (int i = 0; i < MAXI; ++i) {
      const int qq = lane + 32 * i;
      const bool valid = qq < nJ;
      const float w = valid ? wrow[qq] : 0.f;
      const unsigned int key = valid ? key_of<kWanda>(w, __ldg(xnorm + j + qq)) : 0xffffffffu;
      const bool sel = (32 * i < nJ) ? selected<NM>(key, valid, qq, k, c, ctl, nm_n, nm_m) : false;
      const unsigned int bal = __ballot_sync(0xffffffffu, sel);
      const int pos = s + __popc(bal & ((1u << lane) - 1u));
      s += __popc(bal);
      if (valid) mrow[qq] = sel ? 1 : 0;
      if (sel && pos < kCap) {
        Qidx[pos] = qq;
        y[pos] = w;
      }
    }
    if (small_only && s > kNS) return;
    if (s > kNS && !G) {   // excluded by the launcher's choice of scratch
      if (lane == 0) set_error(st, PWP_EINVAL, kSiteSolve);
      return;
    }
    __syncwarp();
    bool ok = true;
    if (s > 0) {
      // after the gather the selected indices are spent: their slots hold 1 / L_ii
      if (s <= kNS) {
        const Rows<true> R{L, nullptr};
        gather_rhat<true>(R, Kt, Qidx, s, B, lane);
        ok = chol_solve<true>(R, y, reinterpret_cast<float*>(Qidx), D, s, lane);
      } else {
        const Rows<false> R{L, G};
        gather_rhat<false>(R, Kt, Qidx, s, B, lane);
        ok = chol_solve<false>(R, y, reinterpret_cast<float*>(Qidx), D, s, lane);
      }
      if (!ok && lane == 0) set_error(st, PWP_ENOTSPD, kSiteSolve);
      if (lane == 0) atomicAdd((unsigned long long*)&ctlp->pruned, (unsigned long long)s);
    }
    float* zrow = Zs + (long long)k * B;
    float* zlo = zrow + (long long)c * B;
    int before = 0;
#pragma unroll
    for (int i = 0; i < MAXI; ++i) {
      const int qq = lane + 32 * i;
      const bool sel = qq < nJ && mrow[qq] != 0;   // this lane's own byte, written above
      const unsigned int bal = __ballot_sync(0xffffffffu, sel);
      const int pos = before + __popc(bal & ((1u << lane) - 1u));
      before += __popc(bal);
      if (qq < B) {
        const float z = (sel && ok) ? y[pos] : 0.f;
        const float h = tf32_head(z);
        zrow[qq] = h;
        zlo[qq] = z - h;
      }
    }
    __syncwarp();
  };
  // First the rows of this warp's slice whose sets exceed the shared rows (the slow
  // general path starts at once, under the other warps' work); then every other row,
  // handed out one at a time, so that a warp held up by a large row takes fewer.
  // (N:M: every row selects B (m - n) / m entries, so when that fits the slab no row can be large)
  const bool any_large = !NM || (long long)B * (nm_m - nm_n) / nm_m > kNS;
  if (any_large)
    for (int k = slot; k < c; k += gridDim.x * nwarps)
      if (count_selected(k) > kNS) solve_row(k, false);
  for (;;) {
    unsigned int k = 0;
    if (lane == 0) k = atomicAdd(&ctlp->row_next, 1u);
    k = __shfl_sync(0xffffffffu, k, 0);
    if (k >= (unsigned int)c) break;
    solve_row((int)k, true);
  }
  // the last warp to run out of rows resets the counters for the next launch
  if (lane == 0) {
    __threadfence();
    if (atomicAdd(&ctlp->warps_done, 1u) == gridDim.x * nwarps - 1) {
      ctlp->row_next = 0u;
      ctlp->warps_done = 0u;
    }
  }
}

// SparseGPT in-block sweep, one warp per row (no shared memory): for each block column
// q in order, e = W_q / U_qq on a selected entry (0 otherwise) and the later block
// columns of the row drop e * U[q, .].  Writes e (the row of E) and the mask.
template <bool NM>
__global__ void __launch_bounds__(256) sparsegpt_solve_kernel(const float* __restrict__ W, int c, int b,
                                                              int j, int B, const float* __restrict__ H,
                                                              const float* __restrict__ udiag,
                                                              Ctl* __restrict__ ctlp, Level2 l2,
                                                              uint8_t* __restrict__ mask,
                                                              float* __restrict__ Zs, int nm_n, int nm_m,
                                                              pwp_stats* st) {
  pdl_enter();
  if (warp_failed(st)) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int k = blockIdx.x * (blockDim.x >> 5) + warp;
  const Ctl ctl = *ctlp;
  clear_used_level2(ctl, l2, blockIdx.x * blockDim.x + threadIdx.x, gridDim.x * blockDim.x);
  if (k >= c) return;
  const int nJ = min(B, b - j);
  constexpr int MAXI = kMaxBlock / 32;
  float w[MAXI], e[MAXI];
  bool sel[MAXI];
  const float* wrow = W + (long long)k * b + j;
  int s = 0;
#pragma unroll
  for (int i = 0; i < MAXI; ++i) {
    const int qq = lane + 32 * i;
    const bool valid = qq < nJ;
    w[i] = valid ? wrow[qq] : 0.f;
    e[i] = 0.f;
    const unsigned int key = valid ? key_of<kObs>(w[i], __ldg(udiag + j + qq)) : 0xffffffffu;
    sel[i] = (32 * i < nJ) ? selected<NM>(key, valid, qq, k, c, ctl, nm_n, nm_m) : false;
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
      if (p == qq) e[i] = ev;
    }
  }
  uint8_t* mrow = mask + (long long)k * b + j;
  float* zrow = Zs + (long long)k * B;
  float* zlo = zrow + (long long)c * B;
#pragma unroll
  for (int i = 0; i < MAXI; ++i) {
    const int qq = lane + 32 * i;
    if (qq < nJ) mrow[qq] = sel[i] ? 1 : 0;
    if (qq < B) {
      const float h = tf32_head(e[i]);
      zrow[qq] = h;
      zlo[qq] = e[i] - h;
    }
  }
  if (lane == 0 && s > 0) atomicAdd((unsigned long long*)&ctlp->pruned, (unsigned long long)s);
}

template <bool NM>
void launch_thanos_variant(const float* W, int c, int b, int j, int B, const float* Kt, const float* xnorm,
                           Ctl* ctl, Level2 l2, uint8_t* mask, float* Zs, int nm_n, int nm_m, float* gscratch,
                           pwp_stats* st, cudaStream_t s) {
  const int smem = kSolveWarps * kPerWarp * 4;
  static std::atomic<unsigned long long> attr_done{0};
  if (first_on_device(attr_done))
    cudaFuncSetAttribute(thanos_solve_kernel<NM>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  const int grid = min((c + kSolveWarps - 1) / kSolveWarps, kSolveCtas);
  launch_pdl(thanos_solve_kernel<NM>, dim3(grid), dim3(kSolveWarps * 32), smem, s, W, c, b, j, B, Kt, xnorm, ctl, l2, mask, Zs, nm_n, nm_m,
                                                               gscratch, st);
}

}  // namespace

// Global scratch of the row solves: one slot per resident warp for factor rows past the
// shared ones, needed only when a row can select more than kNS weights of a block.
size_t solve_scratch_bytes(int c, int B, bool nm, int nm_n, int nm_m) {
  const int smax = nm ? B / nm_m * (nm_m - nm_n) : B;
  if (smax <= kNS) return 0;
  const int grid = min((c + kSolveWarps - 1) / kSolveWarps, kSolveCtas);  // the launch's grid
  return (size_t)grid * kSolveWarps * kGlobalPerWarp * sizeof(float);
}

// A row's selected set is at most min(B, block width) (unstructured) or exactly
// B (m-n)/m (N:M).  8-warp CTAs, two per SM, keep kNS rows of each warp's factor in
// shared memory; rows past them (rows with larger sets) go to the warp's slot of global
// scratch.
int launch_thanos_solve(bool nm, const float* W, int c, int b, int j, int B, const float* Kt,
                        const float* xnorm, Ctl* ctl, Level2 l2, uint8_t* mask, float* Zs, int nm_n, int nm_m,
                        float* gscratch, pwp_stats* st, cudaStream_t s) {
  if (nm)
    launch_thanos_variant<true>(W, c, b, j, B, Kt, xnorm, ctl, l2, mask, Zs, nm_n, nm_m, gscratch, st, s);
  else
    launch_thanos_variant<false>(W, c, b, j, B, Kt, xnorm, ctl, l2, mask, Zs, nm_n, nm_m, gscratch, st, s);
  return 1;
}

int launch_sparsegpt_solve(bool nm, const float* W, int c, int b, int j, int B, const float* H,
                           const float* udiag, Ctl* ctl, Level2 l2, uint8_t* mask, float* Zs, int nm_n, int nm_m,
                           pwp_stats* st, cudaStream_t s) {
  const int grid = (c + 7) / 8;
  if (nm)
    launch_pdl(sparsegpt_solve_kernel<true>, dim3(grid), dim3(256), 0, s, W, c, b, j, B, H, udiag, ctl, l2, mask, Zs, nm_n, nm_m, st);
  else
    launch_pdl(sparsegpt_solve_kernel<false>, dim3(grid), dim3(256), 0, s, W, c, b, j, B, H, udiag, ctl, l2, mask, Zs, nm_n, nm_m, st);
  return 1;
}

}  // namespace pwp
