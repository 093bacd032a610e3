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
// Both phases are blocked by 64-column panels and run in place on the upper
// triangle of H:
//   factor  (panels from the last):  diagonal block in shared memory,
//            panel rows above it via the block's explicit triangular inverse,
//            symmetric rank-64 update of the not-yet-factored top-left part;
//   inverse (panels from the first): U[0:p0, P] = -U[0:p0, 0:p0] V[0:p0, P] U_PP.
#include "pwp_internal.cuh"

namespace pwp {
namespace {

constexpr int NB = kFactorNB;

__global__ void __launch_bounds__(1024) damp_kernel(float* __restrict__ H, int b, float damp,
                                                    float* __restrict__ g_diag, pwp_stats* st) {
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

// Factor the nb x nb diagonal block at p0 (already carrying the updates of every
// later panel): A = V_PP V_PP^T, V_PP upper.  Writes V_PP to H and its inverse
// W_PP = V_PP^-1 (upper, zero below) to Vinv[NB][NB].
__global__ void __launch_bounds__(256) chol_diag_kernel(float* __restrict__ H, int b, int p0, int nb,
                                                        float* __restrict__ Vinv, pwp_stats* st) {
  __shared__ float A[NB][NB + 1];
  __shared__ float Wi[NB][NB + 1];
  __shared__ int bad;
  if (failed(st)) return;
  const int tid = threadIdx.x;
  if (tid == 0) bad = 0;
  for (int idx = tid; idx < nb * nb; idx += blockDim.x) {
    int r = idx / nb, s = idx % nb;
    if (r <= s) {
      float v = H[(long long)(p0 + r) * b + p0 + s];
      A[r][s] = v;
      A[s][r] = v;
    }
  }
  __syncthreads();
  for (int i = nb - 1; i >= 0; --i) {
    if (tid == 0) {
      float d = A[i][i];
      if (!(d > 0.f) || !isfinite(d)) {
        bad = 1;
        set_error(st, PWP_ENOTSPD, kSiteCholDiag);
      } else {
        A[i][i] = sqrtf(d);
      }
    }
    __syncthreads();
    if (bad) return;
    const float piv = A[i][i];
    for (int r = tid; r < i; r += blockDim.x) A[r][i] = A[r][i] / piv;
    __syncthreads();
    for (int idx = tid; idx < i * i; idx += blockDim.x) {
      int r = idx / i, s = idx % i;
      if (r <= s) A[r][s] -= A[r][i] * A[s][i];
    }
    __syncthreads();
  }
  // inverse of the upper-triangular block, one column per thread
  if (tid < nb) {
    const int c = tid;
    for (int r = c + 1; r < NB; ++r) Wi[r][c] = 0.f;
    Wi[c][c] = 1.f / A[c][c];
    for (int i = c - 1; i >= 0; --i) {
      float s = 0.f;
      for (int t = i + 1; t <= c; ++t) s = fmaf(A[i][t], Wi[t][c], s);
      Wi[i][c] = -s / A[i][i];
    }
  }
  __syncthreads();
  for (int idx = tid; idx < NB * NB; idx += blockDim.x) {
    int r = idx / NB, s = idx % NB;
    float w = (r < nb && s < nb && r <= s) ? Wi[r][s] : 0.f;
    Vinv[idx] = w;
    if (r < nb && s < nb && r <= s) H[(long long)(p0 + r) * b + p0 + s] = A[r][s];
  }
}

// Rows above the panel: V[r, P] = A[r, P] (V_PP^T)^-1 = A[r, P] Winv^T, r < p0.
__global__ void __launch_bounds__(256) chol_panel_kernel(float* __restrict__ H, int b, int p0, int nb,
                                                         const float* __restrict__ Vinv,
                                                         const pwp_stats* st) {
  __shared__ float Wi[NB][NB + 1];
  __shared__ float rowbuf[8][NB];
  if (failed(st)) return;
  for (int idx = threadIdx.x; idx < NB * NB; idx += blockDim.x) Wi[idx / NB][idx % NB] = Vinv[idx];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = blockIdx.x * 8 + warp;
  __syncthreads();
  if (r >= p0) return;
  float* hr = H + (long long)r * b + p0;
  for (int t = lane; t < nb; t += 32) rowbuf[warp][t] = hr[t];
  __syncwarp();
  for (int c = lane; c < nb; c += 32) {
    float s = 0.f;
    for (int t = c; t < nb; ++t) s = fmaf(rowbuf[warp][t], Wi[c][t], s);
    hr[c] = s;
  }
}

// Symmetric update of the top-left part: A[r][s] -= sum_t V[r][p0+t] V[s][p0+t],
// r <= s < p0 (64x64 tiles on or above the diagonal).
__global__ void __launch_bounds__(256) chol_update_kernel(float* __restrict__ H, int b, int p0, int nb,
                                                          const pwp_stats* st) {
  __shared__ float Ar[64][NB + 1];
  __shared__ float Br[64][NB + 1];
  if (failed(st)) return;
  const int nT = (p0 + 63) / 64;
  int I = 0, rem = blockIdx.x;
  while (rem >= nT - I) { rem -= nT - I; ++I; }
  const int J = I + rem;
  const int i0 = I * 64, j0 = J * 64;
  for (int idx = threadIdx.x; idx < 64 * NB; idx += blockDim.x) {
    int rr = idx / NB, t = idx % NB;
    float a = 0.f, c = 0.f;
    if (t < nb) {
      if (i0 + rr < p0) a = H[(long long)(i0 + rr) * b + p0 + t];
      if (j0 + rr < p0) c = H[(long long)(j0 + rr) * b + p0 + t];
    }
    Ar[rr][t] = a;
    Br[rr][t] = c;
  }
  __syncthreads();
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4] = {};
  for (int t = 0; t < nb; ++t) {
    float av[4], bv[4];
#pragma unroll
    for (int x = 0; x < 4; ++x) av[x] = Ar[ty + 16 * x][t];
#pragma unroll
    for (int y = 0; y < 4; ++y) bv[y] = Br[tx + 16 * y][t];
#pragma unroll
    for (int x = 0; x < 4; ++x)
#pragma unroll
      for (int y = 0; y < 4; ++y) acc[x][y] = fmaf(av[x], bv[y], acc[x][y]);
  }
#pragma unroll
  for (int x = 0; x < 4; ++x) {
    int r = i0 + ty + 16 * x;
    if (r >= p0) continue;
#pragma unroll
    for (int y = 0; y < 4; ++y) {
      int s = j0 + tx + 16 * y;
      if (s < p0 && r <= s) H[(long long)r * b + s] -= acc[x][y];
    }
  }
}

// Put every diagonal block's inverse in place (the inverse of an upper-triangular
// matrix has the inverses of its diagonal blocks on its block diagonal).
__global__ void put_diag_inverses_kernel(float* __restrict__ H, int b, const float* __restrict__ Vall,
                                         const pwp_stats* st) {
  if (failed(st)) return;
  const int p = blockIdx.x;
  const int p0 = p * NB, nb = min(NB, b - p0);
  const float* V = Vall + (size_t)p * NB * NB;
  for (int idx = threadIdx.x; idx < NB * NB; idx += blockDim.x) {
    int r = idx / NB, s = idx % NB;
    if (r < nb && s < nb && r <= s) H[(long long)(p0 + r) * b + p0 + s] = V[idx];
  }
}

// T[r][c] = sum_{t = r}^{p0-1} U[r][t] V[t][p0 + c]  (U: already-inverted top-left
// part, V: factor column block of panel P).  64 rows x nb columns per CTA.
__global__ void __launch_bounds__(256) trmm_kernel(const float* __restrict__ H, int b, int p0, int nb,
                                                   float* __restrict__ T, const pwp_stats* st) {
  __shared__ float Us[64][33];
  __shared__ float Ps[32][NB + 1];
  if (failed(st)) return;
  const int i0 = blockIdx.x * 64;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4] = {};
  for (int t0 = i0; t0 < p0; t0 += 32) {
    for (int idx = threadIdx.x; idx < 64 * 32; idx += blockDim.x) {
      int rr = idx / 32, kk = idx % 32;
      int r = i0 + rr, t = t0 + kk;
      Us[rr][kk] = (r < p0 && t < p0 && t >= r) ? H[(long long)r * b + t] : 0.f;
    }
    for (int idx = threadIdx.x; idx < 32 * NB; idx += blockDim.x) {
      int kk = idx / NB, cc = idx % NB;
      int t = t0 + kk;
      Ps[kk][cc] = (t < p0 && cc < nb) ? H[(long long)t * b + p0 + cc] : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < 32; ++kk) {
      float av[4], bv[4];
#pragma unroll
      for (int x = 0; x < 4; ++x) av[x] = Us[ty + 16 * x][kk];
#pragma unroll
      for (int y = 0; y < 4; ++y) bv[y] = Ps[kk][tx + 16 * y];
#pragma unroll
      for (int x = 0; x < 4; ++x)
#pragma unroll
        for (int y = 0; y < 4; ++y) acc[x][y] = fmaf(av[x], bv[y], acc[x][y]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int x = 0; x < 4; ++x) {
    int r = i0 + ty + 16 * x;
    if (r >= p0) continue;
#pragma unroll
    for (int y = 0; y < 4; ++y) {
      int cc = tx + 16 * y;
      if (cc < nb) T[(long long)r * NB + cc] = acc[x][y];
    }
  }
}

// U[r][p0 + c] = - sum_{t <= c} T[r][t] W_PP[t][c], one row per warp.
__global__ void __launch_bounds__(256) trmm_finish_kernel(float* __restrict__ H, int b, int p0, int nb,
                                                          const float* __restrict__ T,
                                                          const float* __restrict__ Vinv,
                                                          const pwp_stats* st) {
  __shared__ float Wi[NB][NB + 1];
  __shared__ float rowbuf[8][NB];
  if (failed(st)) return;
  for (int idx = threadIdx.x; idx < NB * NB; idx += blockDim.x) Wi[idx / NB][idx % NB] = Vinv[idx];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = blockIdx.x * 8 + warp;
  __syncthreads();
  if (r >= p0) return;
  for (int t = lane; t < nb; t += 32) rowbuf[warp][t] = T[(long long)r * NB + t];
  __syncwarp();
  for (int c = lane; c < nb; c += 32) {
    float s = 0.f;
    for (int t = 0; t <= c; ++t) s = fmaf(rowbuf[warp][t], Wi[t][c], s);
    H[(long long)r * b + p0 + c] = -s;
  }
}

}  // namespace

size_t factor_ws_bytes(int b) {
  size_t np = (size_t)(b + NB - 1) / NB;
  return np * NB * NB * sizeof(float) + (size_t)b * NB * sizeof(float) + 256;
}

cudaError_t launch_damp_factor(float* H, int b, float damp, float* g_diag, void* ws, size_t ws_bytes,
                               pwp_stats* st, cudaStream_t s) {
  const int np = (b + NB - 1) / NB;
  float* Vall = (float*)ws;
  float* T = Vall + (size_t)np * NB * NB;
  long long nl = 0;
  damp_kernel<<<1, 1024, 0, s>>>(H, b, damp, g_diag, st);
  ++nl;
  for (int p = np - 1; p >= 0; --p) {
    const int p0 = p * NB, nb = min(NB, b - p0);
    float* V = Vall + (size_t)p * NB * NB;
    chol_diag_kernel<<<1, 256, 0, s>>>(H, b, p0, nb, V, st);
    ++nl;
    if (p0 > 0) {
      nl += 2;
      chol_panel_kernel<<<(p0 + 7) / 8, 256, 0, s>>>(H, b, p0, nb, V, st);
      const int nT = (p0 + 63) / 64;
      chol_update_kernel<<<nT * (nT + 1) / 2, 256, 0, s>>>(H, b, p0, nb, st);
    }
  }
  put_diag_inverses_kernel<<<np, 256, 0, s>>>(H, b, Vall, st);
  ++nl;
  for (int p = 1; p < np; ++p) {
    const int p0 = p * NB, nb = min(NB, b - p0);
    const float* V = Vall + (size_t)p * NB * NB;
    trmm_kernel<<<(p0 + 63) / 64, 256, 0, s>>>(H, b, p0, nb, T, st);
    trmm_finish_kernel<<<(p0 + 7) / 8, 256, 0, s>>>(H, b, p0, nb, T, V, st);
    nl += 2;
  }
  count_launches(nl);
  return cudaGetLastError();
}

}  // namespace pwp
