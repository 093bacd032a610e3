// The alpha variant: a fraction of the rows kept dense as outliers.
//
// "Pruning LLMs with Thanos", section "Thanos versus SparseGPT on LLaMA-3 8B": the
// alpha = 0.1 variant keeps 10% of the rows as outliers, which lowers the total N:M
// sparsity from 50% to 45%.  The page does not say how the rows are chosen.  Reading used
// here: the floor(alpha * c) rows with the largest sum over q of (W_kq ||X_q||)^2 =
// W_kq^2 G_qq (the squared norm of the row's activation-aware scores; ties: the lower row
// first) stay as they are, and the other rows are pruned as a layer of their own with the
// same configuration.
//
// On the device: the rows' scores (fp64 sums) from W and the diagonal of the undamped H,
// each row's rank by (score descending, row ascending), the kept rows' compact positions;
// the kept rows are gathered into a compact fp32 layer in the workspace, pruned there by
// the ordinary path, and scattered back next to the untouched outlier rows.
#include "pwp_internal.cuh"

namespace pwp {
namespace {

// score[k] = sum_q W_kq^2 H_qq / 2, one warp per row
__global__ void __launch_bounds__(256) row_energy_kernel(const void* __restrict__ W, int wtype, int c, int b,
                                                         const float* __restrict__ H, double* __restrict__ score) {
  pdl_enter();
  const int lane = threadIdx.x & 31;
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, nwarps = (gridDim.x * blockDim.x) >> 5;
  for (int k = warp; k < c; k += nwarps) {
    double sum = 0.0;
    for (int q = lane; q < b; q += 32) {
      const long long i = (long long)k * b + q;
      const float w = wtype == PWP_FP32 ? ((const float*)W)[i]
                                        : __uint_as_float(((unsigned int)((const uint16_t*)W)[i]) << 16);
      sum += (double)w * (double)w * (0.5 * (double)H[(long long)q * b + q]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    if (lane == 0) score[k] = sum;
  }
}

// flag[k] = 1 when fewer than n_out rows precede row k in (score descending, row
// ascending) order; the scores are staged through shared memory in chunks.
__global__ void __launch_bounds__(256) outlier_rank_kernel(const double* __restrict__ score, int c, int n_out,
                                                           int* __restrict__ flag) {
  pdl_enter();
  __shared__ double chunk[1024];
  const int k = blockIdx.x * blockDim.x + threadIdx.x;
  const double sk = k < c ? score[k] : 0.0;
  int rank = 0;
  for (int j0 = 0; j0 < c; j0 += 1024) {
    __syncthreads();
    for (int i = threadIdx.x; i < 1024 && j0 + i < c; i += blockDim.x) chunk[i] = score[j0 + i];
    __syncthreads();
    const int n = min(1024, c - j0);
    for (int i = 0; i < n; ++i) {
      const double sj = chunk[i];
      rank += (sj > sk) || (sj == sk && j0 + i < k);
    }
  }
  if (k < c) flag[k] = rank < n_out ? 1 : 0;
}

// pos[k] = the kept row's index in the compact layer, or -1 for an outlier row (one CTA).
__global__ void __launch_bounds__(1024) compact_positions_kernel(const int* __restrict__ flag, int c,
                                                                 int* __restrict__ pos) {
  pdl_enter();
  __shared__ int warp_sums[32];
  __shared__ int carry;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) carry = 0;
  __syncthreads();
  for (int k0 = 0; k0 < c; k0 += 1024) {
    const int k = k0 + tid;
    const int keep = (k < c && !flag[k]) ? 1 : 0;
    int x = keep;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) warp_sums[warp] = x;
    __syncthreads();
    int before = carry;
    for (int w = 0; w < warp; ++w) before += warp_sums[w];
    if (k < c) pos[k] = keep ? before + x - 1 : -1;
    __syncthreads();
    if (tid == 1023) carry = before + x;
    __syncthreads();
  }
}

__global__ void __launch_bounds__(256) gather_rows_kernel(const void* __restrict__ W, int wtype, int c, int b,
                                                          const int* __restrict__ pos, float* __restrict__ Wc) {
  pdl_enter();
  const long long n = (long long)c * b;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
    const int k = (int)(i / b), q = (int)(i - (long long)k * b);
    const int p = pos[k];
    if (p < 0) continue;
    const float w = wtype == PWP_FP32 ? ((const float*)W)[i]
                                      : __uint_as_float(((unsigned int)((const uint16_t*)W)[i]) << 16);
    Wc[(long long)p * b + q] = w;
  }
}

__global__ void __launch_bounds__(256) scatter_rows_kernel(const void* __restrict__ W, int wtype, int c, int b,
                                                           const int* __restrict__ pos, const float* __restrict__ Wc,
                                                           const uint8_t* __restrict__ mc, float* __restrict__ Wout,
                                                           uint8_t* __restrict__ mask) {
  pdl_enter();
  const long long n = (long long)c * b;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
    const int k = (int)(i / b), q = (int)(i - (long long)k * b);
    const int p = pos[k];
    if (p < 0) {
      Wout[i] = wtype == PWP_FP32 ? ((const float*)W)[i]
                                  : __uint_as_float(((unsigned int)((const uint16_t*)W)[i]) << 16);
      mask[i] = 0;
    } else {
      Wout[i] = Wc[(long long)p * b + q];
      mask[i] = mc[(long long)p * b + q];
    }
  }
}

size_t al256(size_t x) { return (x + 255) & ~(size_t)255; }

}  // namespace

int alpha_rows(const pwp_config* cfg, int c) {
  return cfg->alpha > 0.f ? (int)((double)cfg->alpha * (double)c) : 0;
}

// Workspace of the alpha variant: the compact prune's own workspace, then the compact
// layer (fp32) and mask, the rows' scores, flags and positions.
size_t alpha_ws_bytes(size_t inner, int c, int b, int n_out) {
  const size_t ck = (size_t)(c - n_out);
  return al256(inner) + al256(ck * b * 4) + al256(ck * b) + al256((size_t)c * 8) + 2 * al256((size_t)c * 4);
}

cudaError_t launch_prune_alpha(const pwp_config* cfg, const void* W, int wtype, int c, int b, float* H, float* Wout,
                               uint8_t* mask, void* ws, size_t inner_bytes, pwp_stats* st, cudaStream_t s,
                               bool stats_ready, int n_out,
                               cudaError_t (*inner_prune)(const pwp_config*, const void*, int, int, int, float*,
                                                          float*, uint8_t*, void*, pwp_stats*, cudaStream_t, bool)) {
  const int ck = c - n_out;
  char* base = (char*)ws;
  size_t off = al256(inner_bytes);
  float* Wc = (float*)(base + off);
  off += al256((size_t)ck * b * 4);
  uint8_t* mc = (uint8_t*)(base + off);
  off += al256((size_t)ck * b);
  double* score = (double*)(base + off);
  off += al256((size_t)c * 8);
  int* flag = (int*)(base + off);
  off += al256((size_t)c * 4);
  int* pos = (int*)(base + off);
  const long long n = (long long)c * b;
  const int egrid = (int)min((n + 255) / 256, (long long)8 * kNumSM);
  launch_pdl(row_energy_kernel, dim3(min((c + 7) / 8, 4 * kNumSM)), dim3(256), 0, s, W, wtype, c, b, (const float*)H,
             score);
  launch_pdl(outlier_rank_kernel, dim3((c + 255) / 256), dim3(256), 0, s, (const double*)score, c, n_out, flag);
  launch_pdl(compact_positions_kernel, dim3(1), dim3(1024), 0, s, (const int*)flag, c, pos);
  launch_pdl(gather_rows_kernel, dim3(egrid), dim3(256), 0, s, W, wtype, c, b, (const int*)pos, Wc);
  count_launches(4);
  pwp_config inner = *cfg;
  inner.alpha = 0.f;
  cudaError_t e = inner_prune(&inner, Wc, PWP_FP32, ck, b, H, Wc, mc, ws, st, s, stats_ready);
  if (e != cudaSuccess) return e;
  launch_pdl(scatter_rows_kernel, dim3(egrid), dim3(256), 0, s, W, wtype, c, b, (const int*)pos, (const float*)Wc,
             (const uint8_t*)mc, Wout, mask);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace pwp
