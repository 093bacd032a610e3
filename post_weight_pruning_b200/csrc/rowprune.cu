// No-update baselines: Wanda and magnitude pruning, one output row at a time.
//
// "Weight Pruning in Large Language Models ..." (llms.blog), section "Wanda: Pruning by
// Weights and Activations": the score of W_kq is |W_kq| * ||X_q||_2, the threshold is set
// independently for every output row, the lowest s% of each row are zeroed and no other
// weight changes.  Section "The Failure of Magnitude Pruning in Large Transformers": the
// magnitude baseline ranks by |W_kq| alone (here with the same per-row quota).
//
// A row's floor(s*b) lowest keys (fp32 bit patterns of the scores, as everywhere in this
// library) are found by a four-pass radix select over the row held in shared memory
// (bits 30..23, 22..15, 14..7, 6..0); among keys equal to the threshold the lower columns
// are taken first, counted in column order with warp ballots while the row is written
// out.  N:M: inside every aligned group of m weights the m-n lowest (key, column) go.
// ||X_q|| comes from the undamped H (sqrt(H_qq / 2)) or straight from X ([n, b]) by a
// two-step deterministic reduction (fp64 partial sums over token slices, then the slices
// in order).
#include "pwp_internal.cuh"

namespace pwp {
namespace {

constexpr int kRowThreads = 256;
constexpr int kNormSlices = 32;

__device__ __forceinline__ float load_w(const void* W, int wtype, long long i) {
  return wtype == PWP_FP32 ? reinterpret_cast<const float*>(W)[i]
                           : __uint_as_float(((unsigned int)reinterpret_cast<const uint16_t*>(W)[i]) << 16);
}

__global__ void stats_target_kernel(pwp_stats* st, long long target) {
  st->target = target;
  st->pruned = 0;
}

// ||X_q||^2 partial sums of the token slice blockIdx.y, fp64, one column per thread.
__global__ void __launch_bounds__(256) colnorm_partial_kernel(const void* __restrict__ X, int xtype, long long n,
                                                              int b, double* __restrict__ part) {
  const int q = blockIdx.x * blockDim.x + threadIdx.x;
  if (q >= b) return;
  const long long t0 = n * blockIdx.y / gridDim.y, t1 = n * (blockIdx.y + 1) / gridDim.y;
  double acc = 0.0;
  for (long long t = t0; t < t1; ++t) {
    const float x = load_w(X, xtype, t * b + q);
    acc += (double)x * (double)x;
  }
  part[(long long)blockIdx.y * b + q] = acc;
}

// xnorm[q] = sqrt(sum of the slices in order), or sqrt(H_qq / 2) when H is given.
__global__ void colnorm_finish_kernel(const double* __restrict__ part, int slices, const float* __restrict__ H,
                                      int b, float* __restrict__ xnorm) {
  const int q = blockIdx.x * blockDim.x + threadIdx.x;
  if (q >= b) return;
  if (H) {
    xnorm[q] = sqrtf(0.5f * H[(long long)q * b + q]);
  } else {
    double g = 0.0;
    for (int s = 0; s < slices; ++s) g += part[(long long)s * b + q];
    xnorm[q] = (float)sqrt(g);
  }
}

__device__ __forceinline__ unsigned int row_key(float w, const float* xnorm, int q) {
  return score_key(xnorm ? wanda_score(w, __ldg(xnorm + q)) : fabsf(w));
}

// One row per CTA iteration (persistent grid).  Dynamic shared memory: the row's keys
// and values (2 b words).
__global__ void __launch_bounds__(kRowThreads) row_quota_kernel(const void* __restrict__ W, int wtype, int c, int b,
                                                                const float* __restrict__ xnorm, int quota,
                                                                float* __restrict__ Wout,
                                                                uint8_t* __restrict__ mask, pwp_stats* st) {
  extern __shared__ unsigned int rsm[];
  unsigned int* keys = rsm;
  float* vals = reinterpret_cast<float*>(rsm + b);
  __shared__ unsigned int hist[256];
  __shared__ unsigned int s_prefix, s_rank;
  __shared__ int wtot[kRowThreads / 32];
  if (cta_failed(st)) return;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  unsigned long long removed_here = 0;
  for (int row = blockIdx.x; row < c; row += gridDim.x) {
    const long long base = (long long)row * b;
    for (int q = tid; q < b; q += kRowThreads) {
      const float w = load_w(W, wtype, base + q);
      vals[q] = w;
      keys[q] = row_key(w, xnorm, q);
    }
    if (tid == 0) {
      s_prefix = 0u;
      s_rank = (unsigned int)quota;
    }
    __syncthreads();
    unsigned int T = 0u, m_ties = 0u;
    if (quota > 0 && quota < b) {
      // the quota-th smallest key, eight (last pass seven) bits at a time
      unsigned int himask = 0u;
#pragma unroll 1
      for (int pass = 0; pass < 4; ++pass) {
        const int shift = pass < 3 ? 23 - 8 * pass : 0;
        const unsigned int width_mask = pass < 3 ? 0xffu : 0x7fu;
        hist[tid] = 0u;
        __syncthreads();
        const unsigned int prefix = s_prefix;
        for (int q = tid; q < b; q += kRowThreads) {
          const unsigned int key = keys[q];
          if ((key & himask) == prefix) atomicAdd(&hist[(key >> shift) & width_mask], 1u);
        }
        __syncthreads();
        if (warp == 0) {
          // lane l sums bins 8l..8l+7; the lane whose range holds the rank scans them
          unsigned int sum = 0u;
#pragma unroll
          for (int i = 0; i < 8; ++i) sum += hist[8 * lane + i];
          unsigned int incl = sum;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const unsigned int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
          }
          const unsigned int rank = s_rank;
          const bool here = rank > incl - sum && rank <= incl;
          if (here) {
            unsigned int cum = incl - sum;
            int sel = 8 * lane + 7;
            for (int i = 0; i < 8; ++i) {
              const unsigned int h = hist[8 * lane + i];
              if (rank <= cum + h) {
                sel = 8 * lane + i;
                break;
              }
              cum += h;
            }
            s_prefix = prefix | ((unsigned int)sel << shift);
            s_rank = rank - cum;
          }
        }
        himask |= width_mask << shift;
        __syncthreads();
      }
      T = s_prefix;
      m_ties = s_rank;   // entries equal to T that are taken, in column order
    }
    // write the row; ties at T are counted in column order across rounds of 256
    unsigned int seen = 0u;
    for (int r0 = 0; r0 < b; r0 += kRowThreads) {
      const int q = r0 + tid;
      const bool valid = q < b;
      const unsigned int key = valid ? keys[q] : 0xffffffffu;
      bool rem;
      if (quota >= b) rem = valid;
      else if (quota <= 0) rem = false;
      else rem = valid && key < T;
      const bool tie = valid && quota > 0 && quota < b && key == T;
      const unsigned int bal = __ballot_sync(0xffffffffu, tie);
      if (lane == 0) wtot[warp] = __popc(bal);
      __syncthreads();
      unsigned int before = seen + __popc(bal & ((1u << lane) - 1u));
      unsigned int round_total = 0u;
#pragma unroll
      for (int w = 0; w < kRowThreads / 32; ++w) {
        if (w < warp) before += wtot[w];
        round_total += wtot[w];
      }
      if (tie && before < m_ties) rem = true;
      if (valid) {
        Wout[base + q] = rem ? 0.f : vals[q];
        mask[base + q] = rem ? 1 : 0;
        removed_here += rem ? 1 : 0;
      }
      seen += round_total;
      __syncthreads();  // wtot and the row buffers are reused
    }
  }
  // one atomic per warp
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) removed_here += __shfl_xor_sync(0xffffffffu, removed_here, o);
  if (lane == 0 && removed_here) atomicAdd((unsigned long long*)&st->pruned, removed_here);
}

// N:M: one aligned group of m weights per thread; the m - n lowest (key, column) go.
__global__ void __launch_bounds__(256) group_nm_kernel(const void* __restrict__ W, int wtype, int c, int b,
                                                       const float* __restrict__ xnorm, int nm_n, int nm_m,
                                                       float* __restrict__ Wout, uint8_t* __restrict__ mask,
                                                       pwp_stats* st) {
  if (failed(st)) return;
  const long long groups = (long long)c * (b / nm_m);
  unsigned long long removed_here = 0;
  for (long long g = blockIdx.x * (long long)blockDim.x + threadIdx.x; g < groups;
       g += (long long)gridDim.x * blockDim.x) {
    const long long base = g * nm_m;            // rows are whole groups: b % m == 0
    const int q0 = (int)(base % b);
    float w[32];
    unsigned int key[32];
    for (int e = 0; e < nm_m; ++e) {
      w[e] = load_w(W, wtype, base + e);
      key[e] = row_key(w[e], xnorm, q0 + e);
    }
    for (int e = 0; e < nm_m; ++e) {
      int rank = 0;
      for (int o = 0; o < nm_m; ++o) rank += (key[o] < key[e]) || (key[o] == key[e] && o < e);
      const bool rem = rank < nm_m - nm_n;
      Wout[base + e] = rem ? 0.f : w[e];
      mask[base + e] = rem ? 1 : 0;
      removed_here += rem ? 1 : 0;
    }
  }
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) removed_here += __shfl_xor_sync(0xffffffffu, removed_here, o);
  if (lane == 0 && removed_here) atomicAdd((unsigned long long*)&st->pruned, removed_here);
}

}  // namespace

size_t no_update_ws_bytes(int b) {
  // xnorm (b floats), then the fp64 slice partials, each 256-byte aligned
  const size_t a = ((size_t)b * sizeof(float) + 255) & ~(size_t)255;
  return a + (size_t)kNormSlices * b * sizeof(double) + 256;
}

cudaError_t launch_no_update(const pwp_config* cfg, const void* W, int wtype, int c, int b, const float* H,
                             const void* X, int xtype, long long n, float* Wout, uint8_t* mask, void* ws,
                             pwp_stats* st, bool stats_ready, cudaStream_t s) {
  const bool wanda = cfg->method == PWP_WANDA;
  const bool nm = cfg->pattern == PWP_NM;
  float* xnorm = (float*)ws;
  double* part = (double*)((char*)ws + (((size_t)b * sizeof(float) + 255) & ~(size_t)255));
  long long nl = 0;
  int quota = 0;
  long long target;
  if (nm) {
    target = (long long)c * (b / cfg->nm_m) * (cfg->nm_m - cfg->nm_n);
  } else {
    quota = (int)((double)cfg->sparsity * (double)b);
    target = (long long)c * quota;
  }
  if (!stats_ready) {
    if (cudaMemsetAsync(st, 0, sizeof(pwp_stats), s) != cudaSuccess) return cudaGetLastError();
  }
  stats_target_kernel<<<1, 1, 0, s>>>(st, target);
  ++nl;
  if (wanda) {
    const int gx = (b + 255) / 256;
    prof_begin(kKColNorm, s);
    if (!H) {
      colnorm_partial_kernel<<<dim3(gx, kNormSlices), 256, 0, s>>>(X, xtype, n, b, part);
      ++nl;
    }
    colnorm_finish_kernel<<<gx, 256, 0, s>>>(part, kNormSlices, H, b, xnorm);
    prof_end(kKColNorm, s);
    ++nl;
  }
  int dev = 0, nsm = kNumSM;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  prof_begin(kKRowPrune, s);
  if (nm) {
    const long long groups = (long long)c * (b / cfg->nm_m);
    const int grid = (int)min((groups + 255) / 256, (long long)8 * nsm);
    group_nm_kernel<<<grid, 256, 0, s>>>(W, wtype, c, b, wanda ? xnorm : nullptr, cfg->nm_n, cfg->nm_m, Wout,
                                         mask, st);
  } else {
    const int smem = 2 * b * 4;
    static std::atomic<unsigned long long> attr_done{0};
    if (first_on_device(attr_done))
      cudaFuncSetAttribute(row_quota_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 2 * 16384 * 4);
    // as many resident CTAs as shared memory allows: the radix passes are latency-bound
    int per_sm = 2;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, row_quota_kernel, kRowThreads, smem) != cudaSuccess ||
        per_sm < 1)
      per_sm = 1;
    const long long cap = (long long)per_sm * nsm;
    const int grid = (int)(c < cap ? c : cap);
    row_quota_kernel<<<grid, kRowThreads, smem, s>>>(W, wtype, c, b, wanda ? xnorm : nullptr, quota, Wout, mask,
                                                     st);
  }
  prof_end(kKRowPrune, s);
  ++nl;
  count_launches(nl);
  return cudaGetLastError();
}

}  // namespace pwp
