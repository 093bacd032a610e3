// Hessian accumulation H = beta*H + 2 X X^T, CUDA-core (SIMT fp32) path.
//
// "Weight Pruning in Large Language Models ..." (llms.blog), section "SparseGPT:
// Second-Order Reconstruction at Scale": H = 2 X X^T (damping is added later).
// X is token-major [n, b]; H[i][j] = 2 * sum_t X[t][i] X[t][j].
//
// Only tiles on or above the diagonal are computed; off-diagonal tiles are written
// to both (I, J) and their mirror (J, I), so H comes out fully symmetric.  This
// path serves fp32 activations (where fp32 products must stay exact to fp32
// rounding) and small b; bf16 activations at scale go through the tcgen05 kernel.
#include "pwp_internal.cuh"

namespace pwp {
namespace {

constexpr int TM = 128;   // tile edge (features)
constexpr int TK = 8;     // tokens per smem stage

template <typename T>
__device__ __forceinline__ float ld_as_float(const T* p);
template <>
__device__ __forceinline__ float ld_as_float<float>(const float* p) { return __ldg(p); }
template <>
__device__ __forceinline__ float ld_as_float<uint16_t>(const uint16_t* p) {
  return __uint_as_float(((unsigned int)__ldg(p)) << 16);
}

// blockIdx.x enumerates tile pairs (I <= J) of the upper triangle in row order.
__device__ __forceinline__ void tile_pair(int idx, int nT, int& I, int& J) {
  int i = 0, rem = idx;
  while (rem >= nT - i) { rem -= nT - i; ++i; }
  I = i;
  J = i + rem;
}

template <typename T>
__global__ void __launch_bounds__(256) syrk_simt_kernel(const T* __restrict__ X, long long n, int b,
                                                        float* __restrict__ H, int beta) {
  __shared__ __align__(16) float As[TK][TM];
  __shared__ __align__(16) float Bs[TK][TM];
  const int nT = (b + TM - 1) / TM;
  int I, J;
  tile_pair(blockIdx.x, nT, I, J);
  const int i0 = I * TM, j0 = J * TM;
  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;
  float acc[8][8];
#pragma unroll
  for (int a = 0; a < 8; ++a)
#pragma unroll
    for (int c = 0; c < 8; ++c) acc[a][c] = 0.f;

  // each thread stages 4 elements of As and 4 of Bs per k-chunk
  for (long long t0 = 0; t0 < n; t0 += TK) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      int lin = tid + e * 256;          // 0..1023 over [TK][TM]
      int kk = lin / TM, col = lin % TM;
      long long t = t0 + kk;
      float va = 0.f, vb = 0.f;
      if (t < n) {
        if (i0 + col < b) va = ld_as_float<T>(X + t * b + i0 + col);
        if (j0 + col < b) vb = ld_as_float<T>(X + t * b + j0 + col);
      }
      As[kk][col] = va;
      Bs[kk][col] = vb;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < TK; ++kk) {
      float4 a0 = *reinterpret_cast<const float4*>(&As[kk][ty * 4]);
      float4 a1 = *reinterpret_cast<const float4*>(&As[kk][64 + ty * 4]);
      float4 b0 = *reinterpret_cast<const float4*>(&Bs[kk][tx * 4]);
      float4 b1 = *reinterpret_cast<const float4*>(&Bs[kk][64 + tx * 4]);
      float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int a = 0; a < 8; ++a)
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[a][c] = fmaf(av[a], bv[c], acc[a][c]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int a = 0; a < 8; ++a) {
    int i = i0 + (a < 4 ? ty * 4 + a : 64 + ty * 4 + (a - 4));
    if (i >= b) continue;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      int j = j0 + (c < 4 ? tx * 4 + c : 64 + tx * 4 + (c - 4));
      if (j >= b) continue;
      float v = 2.f * acc[a][c];
      float* p = H + (long long)i * b + j;
      *p = beta ? *p + v : v;
      if (I != J) {
        float* q = H + (long long)j * b + i;
        *q = beta ? *q + v : v;
      }
    }
  }
}

}  // namespace

cudaError_t launch_hessian_simt(const void* X, int xtype, long long n, int b, float* H, int beta,
                                cudaStream_t s) {
  int nT = (b + TM - 1) / TM;
  int pairs = nT * (nT + 1) / 2;
  if (xtype == PWP_FP32)
    syrk_simt_kernel<float><<<pairs, 256, 0, s>>>((const float*)X, n, b, H, beta);
  else
    syrk_simt_kernel<uint16_t><<<pairs, 256, 0, s>>>((const uint16_t*)X, n, b, H, beta);
  return cudaGetLastError();
}

}  // namespace pwp
