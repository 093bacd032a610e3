// Compressed 2:4 storage of a pruned layer.
//
// "Weight Pruning in Large Language Models ..." (llms.blog), section "N:M Semi-Structured
// Sparsity (2:4 Pattern)": in every aligned group of four weights of a row two are kept,
// and only those two values (16-bit) and their 2-bit positions are stored.  The pages do
// not give the metadata layout the tensor cores read; here each group's positions form
// one 4-bit field idx0 | idx1 << 2 (idx0 < idx1), eight groups per 32-bit word, the first
// group in the lowest bits, words row-major; values are bfloat16 (round to nearest even)
// in column order.  One thread per metadata word (eight groups).
#include <cuda_bf16.h>

#include "pwp_internal.cuh"

namespace pwp {
namespace {

__global__ void __launch_bounds__(256) pack24_kernel(const float* __restrict__ What, const uint8_t* __restrict__ mask,
                                                     int c, int b, uint16_t* __restrict__ values,
                                                     uint32_t* __restrict__ meta, pwp_stats* st) {
  const int groups = b / 4, words = (groups + 7) / 8;
  const long long total = (long long)c * words;
  for (long long t = blockIdx.x * (long long)blockDim.x + threadIdx.x; t < total;
       t += (long long)gridDim.x * blockDim.x) {
    const int k = (int)(t / words), wd = (int)(t - (long long)k * words);
    uint32_t word = 0u;
    for (int i = 0; i < 8; ++i) {
      const int g = 8 * wd + i;
      if (g >= groups) break;
      const long long at = (long long)k * b + 4 * g;
      const uchar4 m4 = *reinterpret_cast<const uchar4*>(mask + at);
      const float4 w4 = *reinterpret_cast<const float4*>(What + at);
      const bool keep[4] = {m4.x == 0, m4.y == 0, m4.z == 0, m4.w == 0};
      auto pick = [&](int e) { return e == 0 ? w4.x : e == 1 ? w4.y : e == 2 ? w4.z : w4.w; };
      int idx[2] = {0, 0}, nk = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e)
        if (keep[e]) {
          if (nk < 2) idx[nk] = e;
          ++nk;
        }
      if (nk != 2) {   // not a 2:4 pattern
        set_error(st, PWP_EINVAL, kSitePack);
        idx[0] = 0;
        idx[1] = 1;
      }
      const long long vo = (long long)k * (2 * groups) + 2 * g;
      values[vo] = __bfloat16_as_ushort(__float2bfloat16_rn(pick(idx[0])));
      values[vo + 1] = __bfloat16_as_ushort(__float2bfloat16_rn(pick(idx[1])));
      word |= (uint32_t)(idx[0] | (idx[1] << 2)) << (4 * i);
    }
    meta[t] = word;
  }
}

}  // namespace

cudaError_t launch_pack24(const float* What, const uint8_t* mask, int c, int b, uint16_t* values, uint32_t* meta,
                          pwp_stats* st, cudaStream_t s) {
  const long long words = (long long)c * ((b / 4 + 7) / 8);
  const int grid = (int)min((words + 255) / 256, (long long)8 * kNumSM);
  pack24_kernel<<<grid > 0 ? grid : 1, 256, 0, s>>>(What, mask, c, b, values, meta, st);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace pwp
