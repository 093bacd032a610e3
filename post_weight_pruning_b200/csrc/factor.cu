// Damping and factorisation of the layer Hessian.
//
// Goal: U upper triangular with (H + lambda I)^-1 = U^T U, i.e. the Cholesky factor
// of the inverse Hessian that "Weight Pruning in Large Language Models ..."
// (llms.blog, section "SparseGPT: Second-Order Reconstruction at Scale") computes
// once per layer.  Row j of U carries the inverse Hessian of the problem in which
// the columns before j are frozen, which is what both the column-sequential and the
// block (Thanos) updates need ("Pruning LLMs with Thanos", section "The scaling
// problem, and what SparseGPT changes").
//
// Route, without ever forming H^-1:  H_d = V V^T with V upper triangular (a Cholesky
// factorisation that starts from the last column), then U = V^-1.  Because
// H_d^-1 = V^-T V^-1 = U^T U with U upper, this is the required factor.
// Both phases run in place on the upper triangle of H:
//   factor, 64-column panels from the last: rows above the panel via the diagonal
//     block's explicit inverse, then a symmetric rank-64 update of the top-left part
//     on the tensor cores (the 3xTF32 update kernel, tiles on or above the diagonal),
//     then the next panel's diagonal block, factored and inverted by one CTA; where TMA
//     cannot take the shape, a CUDA-core update whose CTA holding the next diagonal
//     block also factors and inverts it (look-ahead);
//   inverse, recursive doubling: with the diagonal blocks inverted, neighbouring
//     blocks [A B; 0 D] are merged as [A^-1, -A^-1 B D^-1; 0, D^-1] level by level,
//     each level two batched triangular-times-dense products.
#include "tc_common.cuh"

namespace pwp {
namespace {

constexpr int NB = kFactorNB;  // 64
constexpr int kDiagThreads = 256;

__global__ void __launch_bounds__(1024) damp_kernel(float* __restrict__ H, int b, float damp,
                                                    float* __restrict__ g_diag, pwp_stats* st) {
  pdl_enter();
  __shared__ double red[32];
  __shared__ float lam_s;
  double s = 0.0;
  for (int q = threadIdx.x; q < b; q += blockDim.x) {
    float h = H[(long long)q * b + q];
    s += (double)h;
    g_diag[q] = 0.5f * h;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_down_sync(0xffffffffu, s, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x < 32) {
    double v = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.0;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_down_sync(0xffffffffu, v, o);
    if (threadIdx.x == 0) {
      lam_s = (float)((double)damp * (v / (double)b));
      st->lambda = lam_s;
    }
  }
  __syncthreads();
  const float lam = lam_s;
  for (int q = threadIdx.x; q < b; q += blockDim.x) H[(long long)q * b + q] += lam;
}

// Cholesky of an 8 x 8 SPD block in registers (lower triangle; compile-time indices
// throughout): L L^T = D, with L's diagonal the pivots' square roots and il their
// reciprocals.  False on a non-positive or non-finite pivot.
__device__ __forceinline__ bool chol8(float (&L)[8][8], float (&il)[8]) {
  bool ok = true;
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    const float piv = L[c][c];
    ok = ok && (piv > 0.f) && isfinite(piv);
    il[c] = rsqrtf(piv);
    L[c][c] = piv * il[c];
#pragma unroll
    for (int r = c + 1; r < 8; ++r) L[r][c] *= il[c];
#pragma unroll
    for (int r = c + 1; r < 8; ++r)
#pragma unroll
      for (int c2 = c + 1; c2 <= r; ++c2) L[r][c2] = fmaf(-L[r][c], L[c2][c], L[r][c2]);
  }
  return ok;
}

// Factor the nb x nb diagonal block (nb <= 64) held in A (symmetric; the upper triangle
// is read) as A = V V^T with V upper triangular, and invert V.  256 threads.  Working on
// the reversed matrix P = J A J (J the reversal; P[r][c] = A[63-r][63-c], so P's lower
// triangle is A's upper one and the work happens in place), this is the ordinary
// Cholesky P = L L^T from the top-left, with V = J L J and V^-1 = J X J for X = L^-1.
// Right-looking in 8-column steps, with X built alongside by forward elimination from
// X = I.  Per step k (columns blk = [8k, 8k+8), rows below from r0 = 8k+8):
//   (b) threads 0..63: thread r < 56-8k forms row r0+r of the panel, L[i, blk] =
//       P[i, blk] L_kk^-T (forward substitution with the factored diagonal block), the
//       others bring column t < r0 of the block's rows of X up to date, X[blk, t] :=
//       L_kk^-1 X[blk, t] (the block's own columns start as I and become L_kk^-1);
//   (c) warp 0 applies the step to the next diagonal block and factors it (look-ahead:
//       step k+1's 8x8 Cholesky runs under the rest of step k), while warps 1..7 update
//       the rest of the trailing part, P[i][j] -= L[i, blk] L[j, blk], and eliminate the
//       block's rows from X's rows below it, X[i][t] -= L[i, blk] X[blk, t], t < r0, in
//       2x2 register tiles.
// Two barriers per step.  On entry A's upper triangle holds the block with rows and
// columns beyond nb (A indices >= nb) an identity pad, Wi = I and *bad = 0, visible to
// every thread (load_diag_block).  On return A's upper triangle holds V and Wi holds V^-1
// (upper, zero below).  Returns false on a non-positive pivot (recorded in st).
__device__ bool factor_diag_block(float (*A)[NB + 1], float (*Wi)[NB + 1], int nb, int* bad, pwp_stats* st) {
  constexpr int BS = 8, NBK = NB / BS, LD = NB + 1;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  __shared__ float il_s[NB];
  float* const Pe = &A[NB - 1][NB - 1];   // P(r, c) = Pe[-(r * LD + c)]
  float* const Xe = &Wi[NB - 1][NB - 1];
  auto P = [&](int r, int c) -> float& { return Pe[-(r * LD + c)]; };
  auto X = [&](int r, int c) -> float& { return Xe[-(r * LD + c)]; };
  (void)nb;
  // warp 0: factor the diagonal block at k0 in place (every lane alike; lane 0 stores)
  auto diag = [&](int k0) {
    float Ld[8][8], il[8];
#pragma unroll
    for (int r = 0; r < 8; ++r)
#pragma unroll
      for (int c = 0; c < 8; ++c) Ld[r][c] = c <= r ? P(k0 + r, k0 + c) : 0.f;
    const bool ok = chol8(Ld, il);
    if (lane == 0) {
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        il_s[k0 + r] = il[r];
#pragma unroll
        for (int c = 0; c <= r; ++c) P(k0 + r, k0 + c) = Ld[r][c];
      }
      if (!ok) *bad = 1;
    }
  };
  // one 2x2 tile of the trailing update of P (rows i0, i0+1; columns j0, j0+1)
  auto ptile = [&](int i0, int j0, int k0) {
    float c00 = P(i0, j0), c01 = P(i0, j0 + 1), c10 = P(i0 + 1, j0), c11 = P(i0 + 1, j0 + 1);
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const float a0 = P(i0, k0 + c), a1 = P(i0 + 1, k0 + c), b0 = P(j0, k0 + c), b1 = P(j0 + 1, k0 + c);
      c00 = fmaf(-a0, b0, c00);
      c01 = fmaf(-a0, b1, c01);
      c10 = fmaf(-a1, b0, c10);
      c11 = fmaf(-a1, b1, c11);
    }
    P(i0, j0) = c00;
    P(i0, j0 + 1) = c01;   // above the diagonal on a diagonal tile: never read
    P(i0 + 1, j0) = c10;
    P(i0 + 1, j0 + 1) = c11;
  };
  if (warp == 0) diag(0);
  __syncthreads();
#pragma unroll 1
  for (int kb = 0; kb < NBK; ++kb) {
    const int k0 = BS * kb, r0 = k0 + BS, rest = NB - r0;
    if (tid < NB) {
      float Ld[8][8], il[8];
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        il[r] = il_s[k0 + r];
#pragma unroll
        for (int c = 0; c < r; ++c) Ld[r][c] = P(k0 + r, k0 + c);
      }
      float x[8];
      if (tid < rest) {                      // panel row r0 + tid
        const int i = r0 + tid;
#pragma unroll
        for (int a2 = 0; a2 < 8; ++a2) {
          float v = P(i, k0 + a2);
#pragma unroll
          for (int c = 0; c < a2; ++c) v = fmaf(-x[c], Ld[a2][c], v);
          x[a2] = v * il[a2];
        }
#pragma unroll
        for (int a2 = 0; a2 < 8; ++a2) P(i, k0 + a2) = x[a2];
      } else {                               // column t of the block's rows of X
        const int t = tid - rest;
#pragma unroll
        for (int a2 = 0; a2 < 8; ++a2) {
          float v = X(k0 + a2, t);
#pragma unroll
          for (int c = 0; c < a2; ++c) v = fmaf(-Ld[a2][c], x[c], v);
          x[a2] = v * il[a2];
        }
#pragma unroll
        for (int a2 = 0; a2 < 8; ++a2) X(k0 + a2, t) = x[a2];
      }
    }
    __syncthreads();
    if (rest > 0) {
      const int th = r0 >> 1;   // first tile row of the trailing part
      if (warp == 0) {
        // the next diagonal block's ten lower 2x2 tiles, then its factorisation
        if (lane < 10) {
          const int ta = lane < 1 ? 0 : lane < 3 ? 1 : lane < 6 ? 2 : 3;
          const int tb = lane - ta * (ta + 1) / 2;
          ptile(r0 + 2 * ta, r0 + 2 * tb, k0);
        }
        __syncwarp();
        diag(r0);
      } else {
        for (int id = tid - 32; id < 32 * 32; id += blockDim.x - 32) {
          const int ti = id >> 5, tj = id & 31;
          if (ti < th || (ti < th + 4 && tj >= th) || tj > ti) continue;
          if (tj >= th) {
            ptile(2 * ti, 2 * tj, k0);
          } else {                           // X rows 2ti, 2ti+1 at columns 2tj, 2tj+1 < r0
            const int i0 = 2 * ti, t0 = 2 * tj;
            float c00 = X(i0, t0), c01 = X(i0, t0 + 1), c10 = X(i0 + 1, t0), c11 = X(i0 + 1, t0 + 1);
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              const float a0 = P(i0, k0 + c), a1 = P(i0 + 1, k0 + c), b0 = X(k0 + c, t0), b1 = X(k0 + c, t0 + 1);
              c00 = fmaf(-a0, b0, c00);
              c01 = fmaf(-a0, b1, c01);
              c10 = fmaf(-a1, b0, c10);
              c11 = fmaf(-a1, b1, c11);
            }
            X(i0, t0) = c00;
            X(i0, t0 + 1) = c01;
            X(i0 + 1, t0) = c10;
            X(i0 + 1, t0 + 1) = c11;
          }
        }
      }
    }
    __syncthreads();
  }
  // a non-positive pivot anywhere (the steps after it ran on garbage, harmlessly)
  if (*bad) {
    if (tid == 0) set_error(st, PWP_ENOTSPD, kSiteCholDiag);
    return false;
  }
  return true;
}

// The block at (q0, q0) of H into A (upper triangle; identity pad beyond nb), Wi = I and
// *bad = 0, then a barrier.  256 threads: thread t owns column t % 64 and rows t / 64 + 4m,
// its sixteen loads all in flight at once.
__device__ __forceinline__ void load_diag_block(const float* H, int b, int q0, int nb, float (*A)[NB + 1],
                                                float (*Wi)[NB + 1], int* bad) {
  const int tid = threadIdx.x, sc = tid & (NB - 1), r0 = tid >> 6;
  float v[NB * NB / 256];
#pragma unroll
  for (int m = 0; m < NB * NB / 256; ++m) {
    const int r = r0 + 4 * m;
    v[m] = (r == sc) ? 1.f : 0.f;
    if (r <= sc && sc < nb) v[m] = H[(long long)(q0 + r) * b + q0 + sc];
  }
#pragma unroll
  for (int m = 0; m < NB * NB / 256; ++m) {
    const int r = r0 + 4 * m;
    if (r <= sc) A[r][sc] = v[m];
    Wi[r][sc] = (r == sc) ? 1.f : 0.f;
  }
  if (tid == 0) *bad = 0;
  __syncthreads();
}

// V (A's upper triangle) back into H's block and V^-1 (upper, zero below) into Vinv,
// 64 x 64 row-major (zero outside nb x nb).
__device__ __forceinline__ void store_diag_block(float* H, int b, int q0, int nb, float (*A)[NB + 1],
                                                 float (*Wi)[NB + 1], float* __restrict__ Vinv) {
  const int tid = threadIdx.x, sc = tid & (NB - 1), r0 = tid >> 6;
#pragma unroll
  for (int m = 0; m < NB * NB / 256; ++m) {
    const int r = r0 + 4 * m;
    const bool in = r <= sc && sc < nb;
    Vinv[r * NB + sc] = in ? Wi[r][sc] : 0.f;
    if (in) H[(long long)(q0 + r) * b + q0 + sc] = A[r][sc];
  }
}

// Stand-alone factorisation of the diagonal block at p0 (used for the last panel, and for
// every panel when the trailing update runs on the tensor cores): one CTA of 256 threads.
__global__ void __launch_bounds__(kDiagThreads) chol_diag_kernel(float* __restrict__ H, int b, int p0, int nb,
                                                        float* __restrict__ Vinv, pwp_stats* st) {
  pdl_enter();
  extern __shared__ __align__(16) float dsm[];   // A and Wi, 2 x NB x (NB + 1) floats
  float (*A)[NB + 1] = reinterpret_cast<float (*)[NB + 1]>(dsm);
  float (*Wi)[NB + 1] = reinterpret_cast<float (*)[NB + 1]>(dsm + NB * (NB + 1));
  __shared__ int bad;
  if (cta_failed(st)) return;
  load_diag_block(H, b, p0, nb, A, Wi, &bad);
  if (!factor_diag_block(A, Wi, nb, &bad, st)) return;
  store_diag_block(H, b, p0, nb, A, Wi, Vinv);
}

// The next panel's diagonal block, off the factor's critical path.  Between the trailing
// update of panel p+1 and the end of the factor nothing changes the block [q0, q0+64)^2,
// q0 = p0 - 64 (panel p's update leaves it as it was), nor the pre-panel values Ar of rows
// q0..q0+63 in panel p's columns (panel p parks their V in a slot, the next panel puts it in
// place), so this kernel runs on a side stream beside panel p and its update: A = S - Vr Vr^T
// with S the block and Vr = Ar V_PP^-T (the same products, in the same order, as the panel
// kernel's), then factored and inverted as in chol_diag_kernel, V^-1 into the block's slot
// of Vinv.  V itself is not stored: nothing reads H's diagonal blocks before they receive
// their inverses (put_diag_inverses_kernel).
__global__ void __launch_bounds__(kDiagThreads) chol_diag_ahead_kernel(const float* __restrict__ H, int b,
                                                                       int p0, int nb,
                                                                       const float* __restrict__ Vinv_p,
                                                                       float* __restrict__ Vinv, pwp_stats* st) {
  pdl_enter();
  extern __shared__ __align__(16) float dsm[];   // three 64 x 65 arrays
  float (*A)[NB + 1] = reinterpret_cast<float (*)[NB + 1]>(dsm);
  float (*Wi)[NB + 1] = reinterpret_cast<float (*)[NB + 1]>(dsm + NB * (NB + 1));
  float (*WpT)[NB + 1] = reinterpret_cast<float (*)[NB + 1]>(dsm + 2 * NB * (NB + 1));
  __shared__ int bad;
  if (cta_failed(st)) return;
  const int q0 = p0 - NB, tid = threadIdx.x, sc = tid & (NB - 1), r0 = tid >> 6;
  {
    // S into A's upper triangle, Ar into Wi, V_PP^-1 transposed into WpT: loads in flight
    float v[NB * NB / 256], w[NB * NB / 256], x[NB * NB / 256];
#pragma unroll
    for (int m = 0; m < NB * NB / 256; ++m) {
      const int r = r0 + 4 * m;
      v[m] = r <= sc ? H[(long long)(q0 + r) * b + q0 + sc] : 0.f;
      w[m] = sc < nb ? H[(long long)(q0 + r) * b + p0 + sc] : 0.f;
      x[m] = Vinv_p[r * NB + sc];
    }
#pragma unroll
    for (int m = 0; m < NB * NB / 256; ++m) {
      const int r = r0 + 4 * m;
      if (r <= sc) A[r][sc] = v[m];
      Wi[r][sc] = w[m];
      WpT[sc][r] = x[m];
    }
  }
  __syncthreads();
  {
    // Vr[r][c] = sum_t Ar[r][t] V_PP^-1[c][t], t ascending (the panel kernel's order): row
    // r = tid / 4, columns c = tid % 4 + 4k; results to WpT's place once every thread is done
    const int r = tid >> 2, c0 = tid & 3;
    float acc[NB / 4];
#pragma unroll
    for (int k = 0; k < NB / 4; ++k) acc[k] = 0.f;
#pragma unroll 4
    for (int t = 0; t < NB; ++t) {
      const float a = Wi[r][t];
#pragma unroll
      for (int k = 0; k < NB / 4; ++k) acc[k] = fmaf(a, WpT[t][c0 + 4 * k], acc[k]);
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < NB / 4; ++k) WpT[r][c0 + 4 * k] = acc[k];   // WpT now holds Vr
  }
  __syncthreads();
  {
    // A[r][c] -= sum_t Vr[r][t] Vr[c][t] for r <= c: one 4 x 4 tile per thread (tiles on
    // or above the diagonal of a 16 x 16 tile grid)
    const int tr = tid >> 4, tc = tid & 15;
    if (tr <= tc) {
      float acc[4][4] = {};
#pragma unroll 4
      for (int t = 0; t < NB; ++t) {
        float a[4], c4[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          a[i] = WpT[4 * tr + i][t];
          c4[i] = WpT[4 * tc + i][t];
        }
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], c4[j], acc[i][j]);
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if (4 * tr + i <= 4 * tc + j) A[4 * tr + i][4 * tc + j] -= acc[i][j];
    }
  }
#pragma unroll
  for (int m = 0; m < NB * NB / 256; ++m) {
    const int r = r0 + 4 * m;
    Wi[r][sc] = (r == sc) ? 1.f : 0.f;
  }
  if (tid == 0) bad = 0;
  __syncthreads();
  if (!factor_diag_block(A, Wi, NB, &bad, st)) return;
#pragma unroll
  for (int m = 0; m < NB * NB / 256; ++m) {
    const int r = r0 + 4 * m;
    Vinv[r * NB + sc] = r <= sc ? Wi[r][sc] : 0.f;
  }
}

// Rows above the panel: V[r, P] = A[r, P] (V_PP^T)^-1 = A[r, P] Wi^T, r < p0.  One warp
// per row over a grid of one CTA per SM (the 64x64 inverse is staged once per CTA);
// lane l produces columns l and l + 32.  With vs_hi set, the rows also go to vs_hi /
// vs_lo (row stride NB) as TF32 head and fp32 remainder: the operand of the tensor-core
// trailing update.
__global__ void __launch_bounds__(256) chol_panel_kernel(float* __restrict__ H, int b, int p0, int nb,
                                                         const float* __restrict__ Vinv,
                                                         float* __restrict__ vs_hi, float* __restrict__ vs_lo,
                                                         float* __restrict__ vr_out, const float* __restrict__ vr_in,
                                                         int in_nb, const pwp_stats* st) {
  pdl_enter();
  __shared__ float WiT[NB][NB + 1];  // WiT[t][c] = Wi[c][t]
  __shared__ float rowbuf[8][NB];
  if (cta_failed(st)) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, stride = gridDim.x * 8;
  // each warp's rows go software-pipelined: the next row's two values are loaded before
  // the current row is computed (the first ones before the staging below)
  int r = blockIdx.x * 8 + warp;
  float n0 = 0.f, n1 = 0.f;
  if (r < p0) {
    n0 = lane < nb ? H[(long long)r * b + p0 + lane] : 0.f;
    n1 = lane + 32 < nb ? H[(long long)r * b + p0 + lane + 32] : 0.f;
  }
  {
    // WiT[t][c] = Vinv[c][t]: sixteen loads per thread in flight at once
    float v[NB * NB / 256];
#pragma unroll
    for (int m = 0; m < NB * NB / 256; ++m) v[m] = Vinv[threadIdx.x + 256 * m];
#pragma unroll
    for (int m = 0; m < NB * NB / 256; ++m) {
      const int idx = threadIdx.x + 256 * m;
      WiT[idx % NB][idx / NB] = v[m];
    }
  }
  if (vr_in != nullptr && blockIdx.x == gridDim.x - 1) {
    // the previous panel's rows [p0, p0 + 64), parked in vr_in while this step's diagonal
    // block kernel read their pre-panel values, go into place
    const int sc = threadIdx.x & (NB - 1), r0 = threadIdx.x >> 6;
    float v[NB * NB / 256];
#pragma unroll
    for (int m = 0; m < NB * NB / 256; ++m) v[m] = vr_in[(r0 + 4 * m) * NB + sc];
    if (sc < in_nb) {
#pragma unroll
      for (int m = 0; m < NB * NB / 256; ++m) H[(long long)(p0 + r0 + 4 * m) * b + p0 + NB + sc] = v[m];
    }
  }
  __syncthreads();
  const int q0 = vr_out != nullptr ? p0 - NB : p0;   // rows from q0 on are parked in vr_out
  for (; r < p0; r += stride) {
    float* hr = H + (long long)r * b + p0;
    rowbuf[warp][lane] = n0;
    rowbuf[warp][lane + 32] = n1;
    const int rn = r + stride;
    if (rn < p0) {
      n0 = lane < nb ? H[(long long)rn * b + p0 + lane] : 0.f;
      n1 = lane + 32 < nb ? H[(long long)rn * b + p0 + lane + 32] : 0.f;
    }
    __syncwarp();
    // Wi is upper triangular: Wi[c][t] = 0 for t < c
    float s0 = 0.f, s1 = 0.f;
#pragma unroll 8
    for (int t = 0; t < NB; ++t) {
      const float x = rowbuf[warp][t];
      s0 = fmaf(x, WiT[t][lane], s0);
      s1 = fmaf(x, WiT[t][lane + 32], s1);
    }
    float* dst = r < q0 ? hr : vr_out + (r - q0) * NB;
    if (lane < nb) dst[lane] = s0;
    if (lane + 32 < nb) dst[lane + 32] = s1;
    if (vs_hi) {
      const float h0 = tf32_head(s0), h1 = tf32_head(s1);
      vs_hi[(size_t)r * NB + lane] = h0;
      vs_lo[(size_t)r * NB + lane] = s0 - h0;
      vs_hi[(size_t)r * NB + lane + 32] = h1;
      vs_lo[(size_t)r * NB + lane + 32] = s1 - h1;
    }
    __syncwarp();
  }
}

// Symmetric update of the top-left part on the CUDA cores (when the tensor-core update
// cannot take the shape): A[r][s] -= sum_t V[r][p0+t] V[s][p0+t] for r <= s < p0,
// 128x128 tiles on or above the diagonal, 8x8 outputs per thread; with keep >= 0 the block
// [keep, p0)^2 is left as it was and the panel's rows from keep on are read from vr, where
// the panel kernel parked them.
__global__ void __launch_bounds__(256) chol_update_kernel(float* __restrict__ H, int b, int p0, int nb, int keep,
                                                          const float* __restrict__ vr, const pwp_stats* st) {
  pdl_enter();
  extern __shared__ __align__(16) float fsm[];
  float (*As)[128 + 4] = reinterpret_cast<float (*)[132]>(fsm);               // [NB][132], k-major
  float (*Bs)[128 + 4] = reinterpret_cast<float (*)[132]>(fsm + NB * 132);
  if (cta_failed(st)) return;
  const int nT = (p0 + 127) / 128;
  int I = 0, rem = blockIdx.x;
  while (rem >= nT - I) { rem -= nT - I; ++I; }
  const int J = I + rem;
  const int i0 = I * 128, j0 = J * 128;
  for (int idx = threadIdx.x; idx < 128 * NB; idx += blockDim.x) {
    const int rr = idx / NB, t = idx % NB;
    float a = 0.f, c = 0.f;
    if (t < nb) {
      // the panel rows from keep on are parked in vr (64 x 64), the others are in place
      const int ri = i0 + rr, rj = j0 + rr;
      if (ri < p0) a = (keep >= 0 && ri >= keep) ? vr[(ri - keep) * NB + t] : H[(long long)ri * b + p0 + t];
      if (rj < p0) c = (keep >= 0 && rj >= keep) ? vr[(rj - keep) * NB + t] : H[(long long)rj * b + p0 + t];
    }
    As[t][rr] = a;
    Bs[t][rr] = c;
  }
  __syncthreads();
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[8][8] = {};
#pragma unroll 4
  for (int t = 0; t < NB; ++t) {
    const float4 a0 = *reinterpret_cast<const float4*>(&As[t][ty * 4]);
    const float4 a1 = *reinterpret_cast<const float4*>(&As[t][64 + ty * 4]);
    const float4 b0 = *reinterpret_cast<const float4*>(&Bs[t][tx * 4]);
    const float4 b1 = *reinterpret_cast<const float4*>(&Bs[t][64 + tx * 4]);
    const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
    const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
    for (int x = 0; x < 8; ++x)
#pragma unroll
      for (int y = 0; y < 8; ++y) acc[x][y] = fmaf(av[x], bv[y], acc[x][y]);
  }
#pragma unroll
  for (int x = 0; x < 8; ++x) {
    const int r = i0 + (x < 4 ? ty * 4 + x : 64 + ty * 4 + x - 4);
    if (r >= p0) continue;
#pragma unroll
    for (int y = 0; y < 8; ++y) {
      const int s = j0 + (y < 4 ? tx * 4 + y : 64 + tx * 4 + y - 4);
      if (s < p0 && r <= s && !(r >= keep && keep >= 0)) H[(long long)r * b + s] -= acc[x][y];
    }
  }
}

// Put every diagonal block's inverse in place (the inverse of an upper-triangular
// matrix has the inverses of its diagonal blocks on its block diagonal).
__global__ void put_diag_inverses_kernel(float* __restrict__ H, int b, const float* __restrict__ Vall,
                                         const float* __restrict__ vr_last, int last_nb, const pwp_stats* st) {
  pdl_enter();
  if (cta_failed(st)) return;
  if (vr_last != nullptr && blockIdx.x == 0) {
    // the first panel's rows [0, 64), parked by its panel kernel, into place (columns 64..)
    for (int idx = threadIdx.x; idx < NB * NB; idx += blockDim.x) {
      const int rr = idx / NB, cc = idx % NB;
      if (cc < last_nb) H[(long long)rr * b + NB + cc] = vr_last[idx];
    }
  }
  const int p = blockIdx.x;
  const int p0 = p * NB, nb = min(NB, b - p0);
  const float* V = Vall + (size_t)p * NB * NB;
  for (int idx = threadIdx.x; idx < NB * NB; idx += blockDim.x) {
    int r = idx / NB, s = idx % NB;
    if (r < nb && s < nb && r <= s) H[(long long)(p0 + r) * b + p0 + s] = V[idx];
  }
}

// Batched product C = alpha * A B (+ C when accumulate), one 128x128 tile per CTA
// (8x8 per thread), K in chunks of 16.  A (M x K) and B (K x N) are read with row
// stride lda / ldb; a_upper: A is upper triangular (A[m][k] = 0 for k < m);
// b_upper: B is upper triangular (B[k][n] = 0 for n < k).  blockIdx.z selects the
// batch entry, whose matrices start batch_* elements further on.
struct TriGemm {
  int M, N, K;
  const float* A; long long lda, batch_a;
  const float* B; long long ldb, batch_b;
  float* C; long long ldc, batch_c;
  float alpha;
  int a_upper, b_upper;
};

// Operand chunk of one 16-deep K step, held in registers between the global loads and the
// shared-memory stores.  TILE = 128: A rows m0 + (tid >> 2) + 64 h, columns k0 + 4 (tid & 3)
// ..; B rows k0 + (tid >> 5) + 8 h, columns n0 + 4 (tid & 31) ...  TILE = 64: one float4 of
// each (A rows m0 + (tid >> 2); B rows k0 + (tid >> 4), columns n0 + 4 (tid & 15)).
template <int TILE>
struct TriChunk {
  static constexpr int H = TILE / 64;
  float4 a[H], b[H];
};

// vec: every row start and column origin is 16-byte aligned, so whole float4s are read
// and the masks applied afterwards; otherwise element by element.
template <int TILE>
__device__ __forceinline__ void trigemm_load(const TriGemm& g, const float* A, const float* B, int m0, int n0,
                                             int k0, int kend, bool vec, TriChunk<TILE>& ch) {
  constexpr int H = TILE / 64;
  const int tid = threadIdx.x;
#pragma unroll
  for (int h = 0; h < H; ++h) {
    const int m = m0 + (tid >> 2) + 64 * h, k = k0 + 4 * (tid & 3);
    float v[4] = {0.f, 0.f, 0.f, 0.f};
    if (m < g.M) {
      const float* src = A + (long long)m * g.lda + k;
      if (vec && k + 3 < kend) {
        const float4 t = *reinterpret_cast<const float4*>(src);
        v[0] = t.x; v[1] = t.y; v[2] = t.z; v[3] = t.w;
      } else {
#pragma unroll
        for (int e = 0; e < 4; ++e) v[e] = k + e < kend ? src[e] : 0.f;
      }
      if (g.a_upper) {
#pragma unroll
        for (int e = 0; e < 4; ++e) v[e] = k + e >= m ? v[e] : 0.f;   // A[m][k] = 0 for k < m
      }
    }
    ch.a[h] = make_float4(v[0], v[1], v[2], v[3]);
  }
  constexpr int BR = TILE / 4;   // threads per B row
#pragma unroll
  for (int h = 0; h < H; ++h) {
    const int k = k0 + tid / BR + (256 / BR) * h, n = n0 + 4 * (tid % BR);
    float v[4] = {0.f, 0.f, 0.f, 0.f};
    if (k < kend) {
      const float* src = B + (long long)k * g.ldb + n;
      if (vec && n + 3 < g.N) {
        const float4 t = *reinterpret_cast<const float4*>(src);
        v[0] = t.x; v[1] = t.y; v[2] = t.z; v[3] = t.w;
      } else {
#pragma unroll
        for (int e = 0; e < 4; ++e) v[e] = n + e < g.N ? src[e] : 0.f;
      }
      if (g.b_upper) {
#pragma unroll
        for (int e = 0; e < 4; ++e) v[e] = n + e >= k ? v[e] : 0.f;   // B[k][n] = 0 for n < k
      }
    }
    ch.b[h] = make_float4(v[0], v[1], v[2], v[3]);
  }
}

// One TILE x TILE tile of C per CTA of 256 threads, (TILE/16) x (TILE/16) outputs per
// thread (8 x 8 at TILE = 128, 4 x 4 at TILE = 64: four times the CTAs for the narrow
// levels, which would otherwise leave most SMs idle).
template <int TILE>
__global__ void __launch_bounds__(256) trigemm_kernel(TriGemm g, int vec, const pwp_stats* st) {
  constexpr int R = TILE / 16, HALF = TILE / 2;
  pdl_enter();
  __shared__ __align__(16) float As[2][16][TILE + 4];
  __shared__ __align__(16) float Bs[2][16][TILE + 4];
  if (cta_failed(st)) return;
  const float* A = g.A + blockIdx.z * g.batch_a;
  const float* B = g.B + blockIdx.z * g.batch_b;
  float* C = g.C + blockIdx.z * g.batch_c;
  const int m0 = blockIdx.y * TILE, n0 = blockIdx.x * TILE;
  if (m0 >= g.M || n0 >= g.N) return;
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  // the triangular operand bounds the useful k range of this tile
  int kbeg = 0, kend = g.K;
  if (g.a_upper) kbeg = m0;                        // k >= m
  if (g.b_upper) kend = min(kend, n0 + TILE);      // k <= n
  float acc[R][R] = {};
  TriChunk<TILE> ch;
  int buf = 0;
  if (kbeg < kend) trigemm_load<TILE>(g, A, B, m0, n0, kbeg, kend, vec != 0, ch);
  for (int k0 = kbeg; k0 < kend; k0 += 16) {
    // stage the chunk in registers, fetch the next one, then compute on the stage
#pragma unroll
    for (int h = 0; h < TILE / 64; ++h) {
      const int mm = (tid >> 2) + 64 * h, kk = 4 * (tid & 3);
      As[buf][kk][mm] = ch.a[h].x;
      As[buf][kk + 1][mm] = ch.a[h].y;
      As[buf][kk + 2][mm] = ch.a[h].z;
      As[buf][kk + 3][mm] = ch.a[h].w;
      const int kb = tid / (TILE / 4) + (1024 / TILE) * h, nn = 4 * (tid % (TILE / 4));
      *reinterpret_cast<float4*>(&Bs[buf][kb][nn]) = ch.b[h];
    }
    __syncthreads();
    if (k0 + 16 < kend) trigemm_load<TILE>(g, A, B, m0, n0, k0 + 16, kend, vec != 0, ch);
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      float av[R], bv[R];
#pragma unroll
      for (int hh = 0; hh < R / 4; ++hh) {
        const float4 a4 = *reinterpret_cast<const float4*>(&As[buf][kk][HALF * hh + ty * 4]);
        const float4 b4 = *reinterpret_cast<const float4*>(&Bs[buf][kk][HALF * hh + tx * 4]);
        av[4 * hh] = a4.x; av[4 * hh + 1] = a4.y; av[4 * hh + 2] = a4.z; av[4 * hh + 3] = a4.w;
        bv[4 * hh] = b4.x; bv[4 * hh + 1] = b4.y; bv[4 * hh + 2] = b4.z; bv[4 * hh + 3] = b4.w;
      }
#pragma unroll
      for (int x = 0; x < R; ++x)
#pragma unroll
        for (int y = 0; y < R; ++y) acc[x][y] = fmaf(av[x], bv[y], acc[x][y]);
    }
    buf ^= 1;  // the next chunk goes to the other stage: one barrier per chunk suffices
  }
#pragma unroll
  for (int x = 0; x < R; ++x) {
    const int m = m0 + HALF * (x / 4) + ty * 4 + (x & 3);
    if (m >= g.M) continue;
    float* crow = C + (long long)m * g.ldc;
#pragma unroll
    for (int hh = 0; hh < R / 4; ++hh) {
      const int na = n0 + HALF * hh + tx * 4;
      if (vec && na + 3 < g.N) {
        *reinterpret_cast<float4*>(crow + na) = make_float4(g.alpha * acc[x][4 * hh], g.alpha * acc[x][4 * hh + 1],
                                                            g.alpha * acc[x][4 * hh + 2], g.alpha * acc[x][4 * hh + 3]);
      } else {
#pragma unroll
        for (int yy = 0; yy < 4; ++yy)
          if (na + yy < g.N) crow[na + yy] = g.alpha * acc[x][4 * hh + yy];
      }
    }
  }
}

// Operands of the tensor-core levels of the doubling inverse, as TF32 head and fp32
// remainder (the form the 3xTF32 update kernel takes, both K-major).
// split: dst[r][k] = sign * src[r][k] for r < rows, k < cols; with tri, entries left of
// the upper triangle (k + koff < r, k counted from the chunk's first column koff) are 0.
__global__ void __launch_bounds__(256) split_kernel(const float* __restrict__ src, long long lds, int rows, int cols,
                                                    int tri, int koff, float sign, float* __restrict__ hi,
                                                    float* __restrict__ lo, int ldd, const pwp_stats* st) {
  pdl_enter();
  if (failed(st)) return;
  const long long n = (long long)rows * cols;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
    const int r = (int)(i / cols), k = (int)(i - (long long)r * cols);
    float v = src[(long long)r * lds + k];
    if (tri && k + koff < r) v = 0.f;
    v *= sign;
    const float h = tf32_head(v);
    hi[(long long)r * ldd + k] = h;
    lo[(long long)r * ldd + k] = v - h;
  }
}

// Transposed split: dst[q][k] = src[k][q] for k < krows, q < ncols, through 32x32 shared
// tiles (both sides coalesced); with tri, src is upper triangular from the chunk's first row
// koff on: entries with q < k + koff are 0.
__global__ void __launch_bounds__(256) tsplit_kernel(const float* __restrict__ src, long long lds, int krows,
                                                     int ncols, int tri, int koff, float* __restrict__ hi,
                                                     float* __restrict__ lo, int ldd, const pwp_stats* st) {
  pdl_enter();
  __shared__ float tile[32][33];
  if (failed(st)) return;
  const int k0 = blockIdx.y * 32, q0 = blockIdx.x * 32;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;   // 32 x 8
  for (int r = ty; r < 32; r += 8) {
    const int k = k0 + r, q = q0 + tx;
    float v = (k < krows && q < ncols) ? src[(long long)k * lds + q] : 0.f;
    if (tri && q < k + koff) v = 0.f;
    tile[r][tx] = v;
  }
  __syncthreads();
  for (int r = ty; r < 32; r += 8) {
    const int q = q0 + r, k = k0 + tx;
    if (q < ncols && k < krows) {
      const float v = tile[tx][r];
      const float h = tf32_head(v);
      hi[(long long)q * ldd + k] = h;
      lo[(long long)q * ldd + k] = v - h;
    }
  }
}

void launch_trigemm(const TriGemm& g, int batch, const pwp_stats* st, cudaStream_t s) {
  // float4 access needs 16-byte aligned rows and batch entries
  const bool vec = ((uintptr_t)g.A % 16) == 0 && ((uintptr_t)g.B % 16) == 0 && ((uintptr_t)g.C % 16) == 0 &&
                   (g.lda % 4) == 0 && (g.ldb % 4) == 0 && (g.ldc % 4) == 0 && (g.batch_a % 4) == 0 &&
                   (g.batch_b % 4) == 0 && (g.batch_c % 4) == 0;
  const long long tiles128 = (long long)((g.N + 127) / 128) * ((g.M + 127) / 128) * batch;
  if (tiles128 < 2 * kNumSM) {   // too few 128-wide tiles to fill the GPU: 64-wide ones
    dim3 grid((g.N + 63) / 64, (g.M + 63) / 64, batch);
    launch_pdl(trigemm_kernel<64>, grid, dim3(256), 0, s, g, vec ? 1 : 0, st);
  } else {
    dim3 grid((g.N + 127) / 128, (g.M + 127) / 128, batch);
    launch_pdl(trigemm_kernel<128>, grid, dim3(256), 0, s, g, vec ? 1 : 0, st);
  }
}

}  // namespace

// Floats of the doubling levels' temporary: the full pairs of a level, or its ragged
// pair, whichever is larger (the two run one after the other on the stream).
static size_t doubling_tmp_floats(int b) {
  size_t tmp = 0;
  for (size_t m = NB; m < (size_t)b; m *= 2) {
    const size_t full = (size_t)b / (2 * m), rest = (size_t)b - full * 2 * m;
    size_t need = full * m * m;
    if (rest > m && m * (rest - m) > need) need = m * (rest - m);
    if (need > tmp) tmp = need;
  }
  return tmp;
}

// Doubling levels at least this wide run on the tensor cores (3xTF32), their products in
// K chunks of at most kTcChunk; narrower levels stay on the CUDA cores, where the batch of
// small products is latency-bound anyway.
constexpr int kTcLevel = 1024, kTcChunk = 2048;

// The pairs [A B; 0 D] of a doubling level of width m: (first index, width of D).
template <typename F>
static void for_each_pair(int b, int m, F f) {
  const int full = b / (2 * m), rest = b - full * 2 * m;
  for (int p = 0; p < full; ++p) f(p * 2 * m, m);
  if (rest > m) f(full * 2 * m, rest - m);
}

// Floats of the tensor-core levels' scratch: T (m x m2) and the operand chunks (heads and
// remainders, m x KC and m2 x KC), for the largest pair.
static size_t tc_levels_floats(int b) {
  size_t need = 0;
  for (int m = kTcLevel; m < b; m *= 2)
    for_each_pair(b, m, [&](int, int m2) {
      const size_t kc = (size_t)min(kTcChunk, max(m, m2));
      const size_t f = (size_t)m * m2 + 2 * (size_t)m * kc + 2 * (size_t)m2 * kc + 5 * 64;   // + rounding of 5 regions
      if (f > need) need = f;
    });
  return need;
}

// Diagonal-block inverses, two 64 x 64 slots of parked panel rows (the V of the rows that
// form the next diagonal block, held back one step), the doubling temporary, the current panel's rows as
// TF32 head and remainder (2 x b x NB), the last 256-byte aligned, then the tensor-core
// levels' scratch.
size_t factor_ws_bytes(int b) {
  const size_t np = (size_t)(b + NB - 1) / NB;
  return (np * NB * NB + 2 * NB * NB + doubling_tmp_floats(b) + 2 * (size_t)b * NB + tc_levels_floats(b)) *
             sizeof(float) +
         1024;
}

// One pair [A B; 0 D] of a doubling level on the tensor cores: T = A^-1 B, then
// B := -T D^-1, both as W -= Z R on the 3xTF32 update kernel, over K chunks of at most
// kTcChunk (chunk [k0, k1) of A^-1's columns touches only its rows < k1; chunk [k0, k1) of
// D^-1's rows only columns >= k0).  A^-1, B and D^-1 sit in H (row stride b) at (i0, i0),
// (i0, i0+m) and (i0+m, i0+m); the inverses are upper triangular and H's storage left of
// their diagonals is stale, so the operand copies zero it.
static cudaError_t tc_pair(float* H, int b, int i0, int m, int m2, float* tcw, pwp_stats* st, cudaStream_t s,
                           long long* nl) {
  auto al = [](size_t f) { return (f + 63) & ~(size_t)63; };
  const int KC = min(kTcChunk, max(m, m2));
  float* Tm = tcw;
  float* Zh = Tm + al((size_t)m * m2);
  float* Zl = Zh + al((size_t)m * KC);
  float* Rh = Zl + al((size_t)m * KC);
  float* Rl = Rh + al((size_t)m2 * KC);
  float* Ainv = H + (long long)i0 * b + i0;
  float* Bm = Ainv + m;
  float* Dinv = H + (long long)(i0 + m) * b + i0 + m;
  auto split = [&](const float* src, long long lds, int rows, int cols, int tri, int koff, float sign) {
    const long long n = (long long)rows * cols;
    const int grid = (int)min((n + 255) / 256, (long long)8 * kNumSM);
    launch_pdl(split_kernel, dim3(grid), dim3(256), 0, s, src, lds, rows, cols, tri, koff, sign, Zh, Zl, KC,
               (const pwp_stats*)st);
  };
  auto tsplit = [&](const float* src, long long lds, int krows, int ncols, int tri, int koff) {
    launch_pdl(tsplit_kernel, dim3((ncols + 31) / 32, (krows + 31) / 32), dim3(256), 0, s, src, lds, krows, ncols,
               tri, koff, Rh, Rl, KC, (const pwp_stats*)st);
  };
  cudaError_t e = cudaMemsetAsync(Tm, 0, sizeof(float) * (size_t)m * m2, s);
  if (e != cudaSuccess) return e;
  for (int k0 = 0; k0 < m; k0 += KC) {
    const int kc = min(KC, m - k0), rows = min(m, k0 + kc);
    split(Ainv + k0, b, rows, kc, 1, k0, -1.f);                     // Z = -A^-1[:, k0:k1]
    tsplit(Bm + (long long)k0 * b, b, kc, m2, 0, 0);                // R^T = B[k0:k1, :]^T
    if (!launch_stream_tc(kNoScore, Tm, rows, m2, m2, 0, 0, Zh, Zl, kc, KC, Rh, Rl, nullptr, nullptr, m2, nullptr,
                          nullptr, Level2{}, st, s, &e))
      return e != cudaSuccess ? e : cudaErrorNotSupported;
    if (e != cudaSuccess) return e;
    *nl += 3;
  }
  e = cudaMemset2DAsync(Bm, sizeof(float) * (size_t)b, 0, sizeof(float) * (size_t)m2, m, s);
  if (e != cudaSuccess) return e;
  for (int k0 = 0; k0 < m2; k0 += KC) {
    const int kc = min(KC, m2 - k0);
    split(Tm + k0, m2, m, kc, 0, 0, 1.f);                           // Z = T[:, k0:k1]
    tsplit(Dinv + (long long)k0 * b, b, kc, m2, 1, k0);             // R^T = D^-1[k0:k1, :]^T
    if (!launch_stream_tc(kNoScore, Bm, m, m2, b, k0, 0, Zh, Zl, kc, KC, Rh, Rl, nullptr, nullptr, m2, nullptr,
                          nullptr, Level2{}, st, s, &e))
      return e != cudaSuccess ? e : cudaErrorNotSupported;
    if (e != cudaSuccess) return e;
    *nl += 3;
  }
  return cudaSuccess;
}

cudaError_t launch_damp_factor(float* H, int b, float damp, float* g_diag, void* ws, size_t ws_bytes,
                               pwp_stats* st, cudaStream_t s) {
  const int np = (b + NB - 1) / NB;
  float* Vall = (float*)ws;
  float* vrows = Vall + (size_t)np * NB * NB;   // two slots of parked panel rows, by parity
  float* T = vrows + 2 * NB * NB;
  float* vs_hi = reinterpret_cast<float*>(
      (reinterpret_cast<uintptr_t>(T + doubling_tmp_floats(b)) + 255) & ~(uintptr_t)255);
  float* vs_lo = vs_hi + (size_t)b * NB;
  float* tcw = reinterpret_cast<float*>((reinterpret_cast<uintptr_t>(vs_lo + (size_t)b * NB) + 255) & ~(uintptr_t)255);
  static std::atomic<unsigned long long> attr_done{0};
  if (first_on_device(attr_done)) {
    cudaFuncSetAttribute(chol_update_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 2 * NB * 132 * 4);
    cudaFuncSetAttribute(chol_diag_ahead_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         3 * NB * (NB + 1) * 4);
  }
  long long nl = 0;
  launch_pdl(damp_kernel, dim3(1), dim3(1024), 0, s, H, b, damp, g_diag, st);
  ++nl;
  // factor, panels from the last; the last panel's diagonal block stands alone
  {
    const int p = np - 1, p0 = p * NB, nb = b - p0;
    launch_pdl(chol_diag_kernel, dim3(1), dim3(kDiagThreads), 2 * NB * (NB + 1) * 4, s, H, b, p0, nb, Vall + (size_t)p * NB * NB, st);
    ++nl;
  }
  // Each step: on a side stream the next diagonal block's kernel, which reads only what the
  // trailing update of the previous panel left in H (after an event recorded behind it) and
  // the current block's inverse, so it runs beside the panel kernel and this step's update
  // (which leaves that block as it was); the panel, which parks the V of the rows that form
  // the next block and puts the previous step's parked rows in place; the trailing update.
  // The next panel waits for the block's inverse through an event (one of two, by parity,
  // so that waiting for one step's block never waits for the next one's).  While the stream
  // is being captured into a graph everything goes on the stream itself, in the same order.
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  cudaStreamIsCapturing(s, &cap);
  cudaStream_t s2 = s;
  cudaEvent_t ev_upd = nullptr, ev_diag[2] = {nullptr, nullptr};
  if (cap == cudaStreamCaptureStatusNone && np > 1) {
    int lo = 0, hi = 0;
    cudaDeviceGetStreamPriorityRange(&lo, &hi);
    bool ok = cudaStreamCreateWithPriority(&s2, cudaStreamNonBlocking, hi) == cudaSuccess;
    for (cudaEvent_t* ev : {&ev_upd, &ev_diag[0], &ev_diag[1]})
      ok = ok && cudaEventCreateWithFlags(ev, cudaEventDisableTiming) == cudaSuccess;
    if (!ok) {
      if (s2 != s && s2 != nullptr) cudaStreamDestroy(s2);
      for (cudaEvent_t ev : {ev_upd, ev_diag[0], ev_diag[1]})
        if (ev) cudaEventDestroy(ev);
      s2 = s;
      ev_upd = ev_diag[0] = ev_diag[1] = nullptr;
    }
  }
  const bool side = s2 != s;
  cudaError_t e = cudaSuccess;
  for (int p = np - 1; p >= 1 && e == cudaSuccess; --p) {
    const int p0 = p * NB, nb = min(NB, b - p0);
    float* V = Vall + (size_t)p * NB * NB;
    float* Vnext = Vall + (size_t)(p - 1) * NB * NB;
    if (side) {
      e = cudaEventRecord(ev_upd, s);   // behind the previous update (or the last block's factor)
      if (e == cudaSuccess) e = cudaStreamWaitEvent(s2, ev_upd, 0);
      if (e != cudaSuccess) break;
    }
    launch_pdl(chol_diag_ahead_kernel, dim3(1), dim3(kDiagThreads), 3 * NB * (NB + 1) * 4, s2, (const float*)H, b,
               p0, nb, (const float*)V, Vnext, st);
    if (side) {
      e = cudaEventRecord(ev_diag[(p - 1) & 1], s2);
      // this panel needs its own block's inverse (the previous step's side kernel)
      if (e == cudaSuccess && p < np - 1) e = cudaStreamWaitEvent(s, ev_diag[p & 1], 0);
      if (e != cudaSuccess) break;
    }
    const int pgrid = min((p0 + 7) / 8, kNumSM);
    const float* vr_in = p < np - 1 ? vrows + (size_t)((p + 1) & 1) * NB * NB : nullptr;
    const int in_nb = min(NB, b - (p0 + NB));
    launch_pdl(chol_panel_kernel, dim3(pgrid), dim3(256), 0, s, H, b, p0, nb, (const float*)V, vs_hi, vs_lo,
               vrows + (size_t)(p & 1) * NB * NB, vr_in, in_nb, (const pwp_stats*)st);
    // H[0:p0, 0:p0] -= V[0:p0, P] V[0:p0, P]^T on the tensor cores (tiles on or above the
    // diagonal, the next diagonal block left as it is; one SM left to the side kernel), else
    // on the CUDA cores
    cudaError_t e2 = cudaSuccess;
    const bool tc = launch_stream_tc(kNoScore, H, p0, p0, b, 0, 0, vs_hi, vs_lo, nb, NB, vs_hi, vs_lo, nullptr,
                                     nullptr, p0, nullptr, nullptr, Level2{}, st, s, &e2, true, PickArgs{},
                                     side ? 1 : 0, p0 - NB);
    if (e2 != cudaSuccess && e == cudaSuccess) e = e2;
    if (!tc) {
      const int nT = (p0 + 127) / 128;
      launch_pdl(chol_update_kernel, dim3(nT * (nT + 1) / 2), dim3(256), 2 * NB * 132 * 4, s, H, b, p0, nb,
                 p0 - NB, (const float*)(vrows + (size_t)(p & 1) * NB * NB), (const pwp_stats*)st);
    }
    nl += 3;
  }
  // the last block's inverse before the inverses go in place
  if (side && e == cudaSuccess) e = cudaStreamWaitEvent(s, ev_diag[0], 0);
  if (side) {
    for (cudaEvent_t ev : {ev_upd, ev_diag[0], ev_diag[1]}) cudaEventDestroy(ev);
    cudaStreamDestroy(s2);
  }
  if (e != cudaSuccess) return e;
  launch_pdl(put_diag_inverses_kernel, dim3(np), dim3(256), 0, s, H, b, (const float*)Vall,
             np > 1 ? (const float*)(vrows + NB * NB) : nullptr, min(NB, b - NB), (const pwp_stats*)st);
  ++nl;
  // inverse by recursive doubling: merge [A B; 0 D] pairs of width m
  const bool tc_levels = (b % 4) == 0 && tensor_map_encoder() != nullptr;
  for (int m = NB; m < b; m *= 2) {
    if (m >= kTcLevel && tc_levels) {
      cudaError_t ep = cudaSuccess;
      for_each_pair(b, m, [&](int i0, int m2) {
        if (ep != cudaSuccess) return;
        if ((m2 % 4) == 0) {
          ep = tc_pair(H, b, i0, m, m2, tcw, st, s, &nl);
        } else {
          const long long step = (long long)2 * m * b + 2 * m;
          TriGemm g1{m, m2, m, H + (long long)i0 * b + i0, b, step, H + (long long)i0 * b + i0 + m, b, step,
                     T, m2, (long long)m * m2, 1.f, 1, 0};
          launch_trigemm(g1, 1, st, s);
          TriGemm g2{m, m2, m2, T, m2, (long long)m * m2, H + (long long)(i0 + m) * b + i0 + m, b, step,
                     H + (long long)i0 * b + i0 + m, b, step, -1.f, 0, 1};
          launch_trigemm(g2, 1, st, s);
          nl += 2;
        }
      });
      if (ep != cudaSuccess) return ep;
      continue;
    }
    const int full = b / (2 * m);                 // pairs with both halves of width m
    const int rest = b - full * 2 * m;            // a ragged pair if rest > m
    for (int pass = 0; pass < 2; ++pass) {
      int batch, i0, m2;
      if (pass == 0) {
        batch = full;
        i0 = 0;
        m2 = m;
      } else {
        batch = rest > m ? 1 : 0;
        i0 = full * 2 * m;
        m2 = rest - m;
      }
      if (batch == 0) continue;
      const long long step = (long long)2 * m * b + 2 * m;   // next pair's corner
      // T = A^-1 B   (A^-1: m x m upper at (i0, i0); B: m x m2 at (i0, i0+m))
      TriGemm g1{m, m2, m, H + (long long)i0 * b + i0, b, step, H + (long long)i0 * b + i0 + m, b, step,
                 T, m2, (long long)m * m2, 1.f, 1, 0};
      launch_trigemm(g1, batch, st, s);
      // B = -T D^-1  (D^-1: m2 x m2 upper at (i0+m, i0+m))
      TriGemm g2{m, m2, m2, T, m2, (long long)m * m2, H + (long long)(i0 + m) * b + i0 + m, b, step,
                 H + (long long)i0 * b + i0 + m, b, step, -1.f, 0, 1};
      launch_trigemm(g2, batch, st, s);
      nl += 2;
    }
  }
  count_launches(nl);
  return cudaGetLastError();
}

}  // namespace pwp
