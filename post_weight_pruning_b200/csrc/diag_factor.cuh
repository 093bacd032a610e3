// The 64x64 diagonal-block factorisation of the damped Hessian's reverse Cholesky
// (factor.cu has the route and its page citations), shared by the stand-alone kernel and
// the look-ahead CTA of the tensor-core trailing update (stream_tc.cu).
#pragma once

#include "pwp_internal.cuh"

namespace pwp {
namespace diagf {

constexpr int NB = kFactorNB;  // 64

// Cholesky and inverse of an 8 x 8 SPD block in registers (lower triangles; compile-time
// indices throughout): L L^T = D, X = L^-1.  False on a non-positive pivot.
__device__ __forceinline__ bool chol_inv8(float (&L)[8][8], float (&X)[8][8]) {
  bool ok = true;
  float il[8];
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
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    X[r][r] = il[r];
#pragma unroll
    for (int c = 0; c < r; ++c) {
      float acc = 0.f;
#pragma unroll
      for (int t = c; t < r; ++t) acc = fmaf(L[r][t], X[t][c], acc);
      X[r][c] = -il[r] * acc;
    }
  }
  return ok;
}

// Factor the nb x nb diagonal block (nb <= 64) held in A (symmetric; the upper triangle
// is read) as A = V V^T with V upper triangular, and invert V.  At least 64 threads (the
// first 64 take each step's 8x8 block; every other loop is strided by the block size).
// Working on the reversed matrix P = J A J (J the reversal; P[r][s] = A[63-r][63-s], so
// P's lower triangle is A's upper one and the work happens in place), this is the
// ordinary Cholesky P = L L^T from the top-left, with V = J L J and V^-1 = J X J for
// X = L^-1.  Right-looking in 8-column steps, every step two barriers apart:
//   the step's 8 x 8 diagonal block is factored and inverted in registers (Ld, Xd) by
//   each of the first 64 threads alike; thread r < 56 - k0 forms row k0+8+r of the panel,
//   L[i, blk] = P[i, blk] Xd^T; thread t < k0 brings column t of the block's rows of X up
//   to date, X[blk, t] := Xd X[blk, t] (those rows already carry the earlier steps'
//   eliminations; their own columns become Xd);
//   then all threads update the trailing part, P[i][j] -= L[i, blk] L[j, blk], and
//   eliminate the block's rows from X's rows below it, X[i][t] -= L[i, blk] X[blk, t].
// Rows and columns beyond nb (A indices >= nb) are an identity pad.  On return A's upper
// triangle holds V and Wi holds V^-1 (upper, zero below).  Returns false on a
// non-positive pivot (recorded in st).
__device__ inline bool factor_diag_block(float (*A)[NB + 1], float (*Wi)[NB + 1], int nb, int* bad, pwp_stats* st) {
  constexpr int BS = 8, NBK = NB / BS;
  const int tid = threadIdx.x;
  auto P = [&](int r, int c) -> float& { return A[NB - 1 - r][NB - 1 - c]; };
  auto X = [&](int r, int c) -> float& { return Wi[NB - 1 - r][NB - 1 - c]; };
  // identity pad beyond nb (A indices >= nb) and X = 0
  for (int idx = tid; idx < NB * NB; idx += blockDim.x) {
    const int i = idx / NB, jc = idx % NB;
    if (i <= jc && jc >= nb) A[i][jc] = (i == jc) ? 1.f : 0.f;
    Wi[i][jc] = 0.f;
  }
  if (tid == 0) *bad = 0;
  __syncthreads();
#pragma unroll 1
  for (int kb = 0; kb < NBK; ++kb) {
    const int k0 = BS * kb, r0 = k0 + BS, rest = NB - r0;
    if (tid < 64) {
      float Ld[8][8], Xd[8][8];
#pragma unroll
      for (int r = 0; r < 8; ++r)
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          Ld[r][c] = c <= r ? P(k0 + r, k0 + c) : 0.f;
          Xd[r][c] = 0.f;
        }
      const bool ok = chol_inv8(Ld, Xd);
      if (!ok && tid == 0) *bad = 1;
      if (tid < rest) {                      // panel row k0 + 8 + tid
        const int i = r0 + tid;
        float pr[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) pr[c] = P(i, k0 + c);
#pragma unroll
        for (int a = 0; a < 8; ++a) {
          float acc = 0.f;
#pragma unroll
          for (int c = 0; c <= a; ++c) acc = fmaf(pr[c], Xd[a][c], acc);
          P(i, k0 + a) = acc;
        }
      }
      if (tid < k0) {                        // column tid of the block's rows of X
        float xo[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) xo[c] = X(k0 + c, tid);
#pragma unroll
        for (int a = 0; a < 8; ++a) {
          float acc = 0.f;
#pragma unroll
          for (int c = 0; c <= a; ++c) acc = fmaf(Xd[a][c], xo[c], acc);
          X(k0 + a, tid) = acc;
        }
      }
      if (tid == 63) {                       // the block itself
#pragma unroll
        for (int r = 0; r < 8; ++r)
#pragma unroll
          for (int c = 0; c <= r; ++c) {
            P(k0 + r, k0 + c) = Ld[r][c];
            X(k0 + r, k0 + c) = Xd[r][c];
          }
      }
    }
    __syncthreads();
    if (*bad) {
      if (tid == 0) set_error(st, PWP_ENOTSPD, kSiteCholDiag);
      return false;
    }
    // trailing update of P (lower triangle of the rest x rest part) and elimination of
    // the block's rows from the rows of X below it (columns < k0 + 8)
    const int nP = rest * (rest + 1) / 2, nX = rest * r0;
    for (int e = tid; e < nP + nX; e += blockDim.x) {
      if (e < nP) {
        int ii = (int)((sqrtf(8.f * (float)e + 1.f) - 1.f) * 0.5f);
        if ((ii + 1) * (ii + 2) / 2 <= e) ++ii;
        if (ii * (ii + 1) / 2 > e) --ii;
        const int i = r0 + ii, j = r0 + (e - ii * (ii + 1) / 2);
        float acc = P(i, j);
#pragma unroll
        for (int c = 0; c < 8; ++c) acc = fmaf(-P(i, k0 + c), P(j, k0 + c), acc);
        P(i, j) = acc;
      } else {
        const int e2 = e - nP, i = r0 + e2 / r0, t = e2 % r0;
        float acc = X(i, t);
#pragma unroll
        for (int c = 0; c < 8; ++c) acc = fmaf(-P(i, k0 + c), X(k0 + c, t), acc);
        X(i, t) = acc;
      }
    }
    __syncthreads();
  }
  return true;
}

}  // namespace diagf
}  // namespace pwp
