// Hessian accumulation H = beta*H + 2 X X^T on the 5th-generation tensor cores
// (bf16 activations, fp32 accumulation).
//
// "Weight Pruning in Large Language Models ..." (llms.blog), section "SparseGPT:
// Second-Order Reconstruction at Scale": H = 2 X X^T.  X is token-major [n, b], so
// H[i][j] = 2 sum_t X[t][i] X[t][j] is a product whose two operands are both stored
// feature-contiguous ("MN-major" in the tensor-core operand terminology): A[i][t] =
// X[t][i] and B[t][j] = X[t][j] come straight from X with no transpose.
//
// One CTA computes one 128 x 256 tile of H (rows i0.., columns j0..) over all n tokens:
//   - warp 0 (one thread) issues TMA loads of 64-feature x 64-token boxes (128-byte
//     swizzle) into a 4-stage ring, two boxes for A and four for B per stage;
//   - warp 1 (one thread) issues tcgen05.mma (M=128, N=256, K=16, bf16 x bf16 -> fp32),
//     four per stage, and releases each stage with tcgen05.commit;
//   - warps 2-9 fold the accumulator into fp32 registers and finally write both
//     H[i][j] and its mirror H[j][i] for i <= j, scaled by 2.
// The tensor core's accumulation into tensor memory does not round to nearest: a long
// chain of additions of positive terms (the diagonal of H is a sum of squares) drifts
// low in proportion to the chain's length.  So no accumulator takes more than 512
// tokens: the MMAs of each span of 512 tokens start a fresh accumulator, alternating
// between two 256-column halves of tensor memory, and while the MMAs fill one half the
// epilogue warps add the other, finished half into their running sums (each thread
// holds 128 entries of one tile row) with ordinary round-to-nearest fp32 additions.
// Only tiles that hold some i <= j are launched; entries with i > j are left to their
// mirror, so H comes out exactly symmetric.  Every wait is bounded: a wait that runs
// out records PWP_ETIMEOUT (or, without a status word, writes NaN into the tile), and
// copies and MMAs already in flight are always waited for before the CTA leaves.
#include "tc_common.cuh"

namespace pwp {
namespace {

constexpr int TM = 128, TN = 256, TK = 64, STAGES = 4;
constexpr int SPAN_KT = 8;                       // k-tiles (of TK tokens) per accumulator span
constexpr int BOX_BYTES = 64 * TK * 2;           // one 64-feature x 64-token bf16 box
constexpr int A_BYTES = TM * TK * 2;             // 2 boxes
constexpr int B_BYTES = TN * TK * 2;             // 4 boxes
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;   // 48 KB
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 + 256;
constexpr int kEpiWarps = 8, kThreads = 32 * (2 + kEpiWarps);
constexpr int kCols = TN / 2;                    // tile columns per epilogue thread
// kind::f16 instruction descriptor: D fp32, A and B bf16, both MN-major, N = 256, M = 128
constexpr uint32_t IDESC = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) | (1u << 16) |
                           ((uint32_t)(TN >> 3) << 17) | ((uint32_t)(TM >> 4) << 24);
using namespace tc;

__device__ __forceinline__ void mma_bf16(uint32_t tmem_d, uint64_t da, uint64_t db, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(da), "l"(db), "r"(IDESC), "r"(acc)
      : "memory");
}

// Tiles (I, J) of 128 rows x 256 columns that hold some entry with row <= column,
// enumerated column-tile by column-tile: I < 2J + 2.
__host__ __device__ inline int tile_count(int b) {
  const int nI = (b + TM - 1) / TM, nJ = (b + TN - 1) / TN;
  int cnt = 0;
  for (int J = 0; J < nJ; ++J) cnt += min(nI, 2 * J + 2);
  return cnt;
}

__device__ inline void tile_of(int idx, int b, int& I, int& J) {
  const int nI = (b + TM - 1) / TM;
  J = 0;
  while (true) {
    const int cnt = min(nI, 2 * J + 2);
    if (idx < cnt) break;
    idx -= cnt;
    ++J;
  }
  I = idx;
}

__global__ void __launch_bounds__(kThreads, 1) syrk_tc_kernel(const __grid_constant__ CUtensorMap tmap, long long n,
                                                              int b, float* __restrict__ H, int beta, pwp_stats* st,
                                                              long long spin) {
  pdl_enter();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* afull = empty + STAGES;    // accumulator half a holds a finished span
  uint64_t* aempty = afull + 2;        // accumulator half a has been folded in
  uint64_t* drain = aempty + 2;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;
  volatile int* abortp = &abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int I, J;
  tile_of(blockIdx.x, b, I, J);
  const int i0 = I * TM, j0 = J * TN;
  const int nk = (int)((n + TK - 1) / TK);
  const int nspan = (nk + SPAN_KT - 1) / SPAN_KT;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&afull[a], 1);
      mbar_init(&aempty[a], kEpiWarps);
    }
    mbar_init(drain, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    abort_flag = 0;
  }
  if (warp == 1) tmem_alloc(&tmem_slot, 2 * TN);
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tmem = tmem_slot;

  float acc[kCols];
#pragma unroll
  for (int i = 0; i < kCols; ++i) acc[i] = 0.f;
  bool have = true;

  if (warp == 0) {
    if (lane == 0) {
      prefetch_map(&tmap);
      int issued = 0;
      for (int kt = 0; kt < nk; ++kt) {
        const int s = kt % STAGES;
        if (kt >= STAGES && !mbar_wait(&empty[s], ((kt / STAGES) - 1) & 1, abortp, spin)) {
          *abortp = 1;
          break;
        }
        mbar_expect_tx(&full[s], STAGE_BYTES);
        uint8_t* a = smem + s * STAGE_BYTES;
        uint8_t* bb = a + A_BYTES;
        const int y = kt * TK;
        tma_load_2d(a, &tmap, &full[s], i0, y);
        tma_load_2d(a + BOX_BYTES, &tmap, &full[s], i0 + 64, y);
#pragma unroll
        for (int h = 0; h < 4; ++h) tma_load_2d(bb + h * BOX_BYTES, &tmap, &full[s], j0 + 64 * h, y);
        issued = kt + 1;
      }
      // every copy issued lands before the CTA leaves (already true unless a role gave up)
      for (int kt = issued - STAGES > 0 ? issued - STAGES : 0; kt < issued; ++kt)
        mbar_wait(&full[kt % STAGES], (kt / STAGES) & 1, kDrainLimit);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t sbase = smem_u32(smem);
      bool ok = true;
      for (int kt = 0; kt < nk && ok; ++kt) {
        const int s = kt % STAGES;
        const int sp = kt / SPAN_KT, half = sp & 1;
        const bool first = (kt % SPAN_KT) == 0;
        // a span reuses the half of two spans back once the epilogue has folded it in
        if (first && sp >= 2 && !mbar_wait(&aempty[half], ((sp >> 1) - 1) & 1, abortp, spin)) {
          ok = false;
          break;
        }
        if (!mbar_wait(&full[s], (kt / STAGES) & 1, abortp, spin)) {
          ok = false;
          break;
        }
        fence_after();
        const uint32_t d = tmem + (uint32_t)(half * TN);
        const uint32_t a_addr = sbase + s * STAGE_BYTES;
        const uint32_t b_addr = a_addr + A_BYTES;
#pragma unroll
        for (int kk = 0; kk < TK / 16; ++kk) {
          const uint64_t da = sw128_desc(a_addr + kk * 2048, BOX_BYTES, 1024);
          const uint64_t db = sw128_desc(b_addr + kk * 2048, BOX_BYTES, 1024);
          mma_bf16(d, da, db, (first && kk == 0) ? 0u : 1u);
        }
        mma_commit(&empty[s]);
        if ((kt % SPAN_KT) == SPAN_KT - 1 || kt == nk - 1) mma_commit(&afull[half]);
      }
      if (!ok) *abortp = 1;
      // every MMA issued has finished before tensor memory is released
      mma_commit(drain);
      mbar_wait(drain, 0, kDrainLimit);
    }
    __syncwarp();
  } else {
    // epilogue: warp w reads tensor-memory lanes 32(w%4).. (tile rows) and the tile
    // columns 128 * ((w-2)/4) ..; the running sums of those 128 columns stay in registers
    const int quarter = warp & 3, colh = (warp - 2) >> 2;
    for (int sp = 0; sp < nspan; ++sp) {
      const int half = sp & 1;
      bool ok = mbar_wait(&afull[half], (sp >> 1) & 1, abortp, spin);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) {
        have = false;
        if (lane == 0) *abortp = 1;
        break;
      }
      fence_after();
      const uint32_t base = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(half * TN + colh * kCols);
#pragma unroll
      for (int ch = 0; ch < kCols / 32; ++ch) {
        float v[32];
        tmem_ld32(base + (uint32_t)(ch * 32), v);
#pragma unroll
        for (int i = 0; i < 32; ++i) acc[ch * 32 + i] += v[i];
      }
      fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&aempty[half]);
    }
  }

  fence_before();
  __syncthreads();
  fence_after();
  if (warp == 1) tmem_free(tmem, 2 * TN);
  if (warp < 2) return;

  const bool failed_tile = !have || *abortp;
  const int quarter = warp & 3, colh = (warp - 2) >> 2;
  const int r = i0 + quarter * 32 + lane;
  if (failed_tile) {
    if (threadIdx.x == 64) {
      if (st) set_error(st, PWP_ETIMEOUT, kSiteHessian);
    }
    if (!st && r < b) {
      for (int c = j0 + colh * kCols; c < min(b, j0 + (colh + 1) * kCols); ++c)
        if (r <= c) H[(long long)r * b + c] = __int_as_float(0x7fc00000);
    }
    return;
  }
#pragma unroll
  for (int ch = 0; ch < kCols / 32; ++ch) {
    const int c0 = j0 + colh * kCols + ch * 32;
    if (c0 >= b || r >= b) continue;
    float* v = acc + ch * 32;
    // direct row: this thread's 32 consecutive columns, 16-byte stores where whole
    float* hr = H + (long long)r * b + c0;
    const bool vec = ((b & 3) == 0) && (r <= c0) && (c0 + 32 <= b);
    if (vec) {
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        float4 o = make_float4(2.f * v[4 * q], 2.f * v[4 * q + 1], 2.f * v[4 * q + 2], 2.f * v[4 * q + 3]);
        if (beta) {
          const float4 old = *reinterpret_cast<const float4*>(hr + 4 * q);
          o.x += old.x; o.y += old.y; o.z += old.z; o.w += old.w;
        }
        *reinterpret_cast<float4*>(hr + 4 * q) = o;
        v[4 * q] = o.x; v[4 * q + 1] = o.y; v[4 * q + 2] = o.z; v[4 * q + 3] = o.w;
      }
    } else {
#pragma unroll
      for (int k = 0; k < 32; ++k) {
        const int c = c0 + k;
        if (c < b && r <= c) {
          const float val = beta ? hr[k] + 2.f * v[k] : 2.f * v[k];
          hr[k] = val;
          v[k] = val;
        }
      }
    }
    // mirror: for each column, the warp writes 32 consecutive row entries
#pragma unroll
    for (int k = 0; k < 32; ++k) {
      const int c = c0 + k;
      if (c < b && r < c) H[(long long)c * b + r] = v[k];
    }
  }
}

}  // namespace

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static const PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    return (PFN_cuTensorMapEncodeTiled_v12000) nullptr;
  }();
  return fn;
}

// Declines (used = false) when the shape does not meet the TMA rules (row stride a
// multiple of 16 bytes, 16-byte aligned base) or there is nothing to accumulate.
cudaError_t launch_hessian_tc(const void* X, long long n, int b, float* H, int beta, cudaStream_t s, bool* used,
                              pwp_stats* st) {
  *used = false;
  if (n < 1 || b < 1 || (b % 8) != 0 || ((uintptr_t)X % 16) != 0 || n > 0x7fffffffLL) return cudaSuccess;
  PFN_cuTensorMapEncodeTiled_v12000 encode = tensor_map_encoder();
  if (!encode) return cudaSuccess;
  CUtensorMap map;
  cuuint64_t dims[2] = {(cuuint64_t)b, (cuuint64_t)n};
  cuuint64_t strides[1] = {(cuuint64_t)b * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)TK};
  cuuint32_t estr[2] = {1, 1};
  CUresult cr = encode(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(X), dims, strides, box, estr,
                       CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                       CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (cr != CUDA_SUCCESS) return cudaSuccess;
  static std::atomic<unsigned long long> attr_done{0};
  if (first_on_device(attr_done)) {
    cudaError_t e = cudaFuncSetAttribute(syrk_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
  }
  launch_pdl(syrk_tc_kernel, dim3(tile_count(b)), dim3(kThreads), SMEM_BYTES, s, map, n, b, H, beta, st, wait_limit());
  *used = true;
  return cudaGetLastError();
}

}  // namespace pwp
