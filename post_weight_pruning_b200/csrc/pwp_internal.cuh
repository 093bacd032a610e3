// Internal declarations shared by the CUDA translation units of libpwp.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "../../include/pwp.h"

namespace pwp {

// True on the first call for the current device with this flag word.  Kernel
// attributes (dynamic shared memory limits) are per device, so each device of a
// multi-GPU process sets them once.  Devices past 63 always set them again (harmless).
inline bool first_on_device(std::atomic<unsigned long long>& done) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return true;
  const unsigned long long bit = 1ull << dev;
  return (done.fetch_or(bit) & bit) == 0;
}

// Programmatic dependent launch.  Kernels of the prune's dependent chains are launched
// with programmatic stream serialisation, so a kernel's CTAs may be scheduled while its
// predecessor's last CTAs still run.  Every such kernel therefore starts with pdl_wait()
// (griddepcontrol.wait: the predecessor grid has completed and its writes are visible)
// before it reads anything, and lets its own dependents be scheduled at once
// (pdl_release).  Both are no-ops for a kernel launched without the attribute.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_release() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_enter() {
  pdl_wait();
  pdl_release();
}

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl_plain(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                                    Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// Launch tracing for diagnosis (PWP_TRACE=1 in the environment, read once): every launch
// through launch_pdl prints the kernel's name and shape to stderr, then waits for the
// stream (unless it is being captured) and prints how the kernel ended, so the last line
// names a kernel that does not finish.  Off by default; profile.cu.
bool trace_launches();
void trace_launch(const void* kernel, dim3 grid, dim3 block, size_t smem, cudaStream_t s, cudaError_t launched);

// Launch with programmatic stream serialisation (the kernel must begin with pdl_enter()).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                              Args... args) {
  if (trace_launches()) {
    const cudaError_t e = launch_pdl_plain(kernel, grid, block, smem, s, args...);
    trace_launch(reinterpret_cast<const void*>(kernel), grid, block, smem, s, e);
    return e;
  }
  return launch_pdl_plain(kernel, grid, block, smem, s, args...);
}

constexpr int kNumSM = 148;              // B200
constexpr int kKeyLoBits = 18;           // second radix level: key bits [17:0]
constexpr int kHist1Bits = 31 - kKeyLoBits;  // first level: key bits [30:18] (32 KB of shared memory)
constexpr int kHist1Bins = 1 << kHist1Bits;
constexpr int kHist2Bins = 1 << kKeyLoBits;
constexpr int kHist2SumShift = 9;        // level-2 summary: 512 bins of 512 level-2 bins
constexpr int kHist2SumBins = kHist2Bins >> kHist2SumShift;
constexpr int kFactorNB = 64;            // panel width of the blocked factorisation
constexpr int kMaxBlock = 128;           // largest column block B
constexpr int kSolveCtas = 2 * kNumSM;   // persistent grid of the row-solve kernel
constexpr int kSolveNS = 79;             // factor rows kept in shared memory at capacity 128

// Per-call device control block (lives at the start of the workspace).
struct Ctl {
  long long zstar;        // global removal target (Thanos unstructured)
  long long pruned;       // removals so far
  long long take;         // entries to select in the current region
  long long count_less;   // entries with key < T
  long long m;            // tied entries (key == T) that must also be selected
  long long ties;         // entries with key == T in the region
  long long pstar;        // tie cut-off: column-major position inside the block (inclusive)
  unsigned int b1;        // top-level bin holding the threshold
  unsigned int r1;        // rank of the threshold inside bin b1 (1-based)
  unsigned int T;         // exact 31-bit score key of the threshold
  int mode;               // 0: select nothing, 1: key/position rule
  int b1_valid;           // b1 holds the previous block's level-1 bin: the scoring pass
                          // histograms the low key bits of that bin as it goes
  int l2_ready;           // this block's bin is the predicted one: no re-read needed
  int dirty_pred;         // the predicted level-2 histogram holds counts to clear
  int dirty_reread;       // the re-read level-2 histogram holds counts to clear
  int tie_scan;           // some but not all entries tied at T are taken: locate the cut-off
  unsigned int ticket;    // arrivals of a grid's CTAs; the last one finishes the selection
  unsigned int row_next;  // the row solve's next row to hand out (reset by its last warp)
  unsigned int warps_done;  // the row solve's warps that have run out of rows
};

// Where device-side failures are recorded (pwp_stats::status_site).
enum Site : int {
  kSiteDamp = 1, kSiteCholDiag = 2, kSiteSolve = 3, kSitePick = 4, kSiteFinal = 5, kSiteHessian = 6,
  kSiteStream = 7, kSitePack = 8,
};

__device__ __forceinline__ bool failed(const pwp_stats* st) {
  return *((volatile const int32_t*)&st->status) != PWP_OK;
}

// The early-exit checks below must give every thread of a CTA (or of a warp, for
// kernels that only synchronise within warps) the same answer: another CTA may record
// an error while this one starts, and a thread that returned while its neighbours go
// on to a barrier or a full-mask shuffle would leave them waiting forever.
__device__ __forceinline__ bool cta_failed(const pwp_stats* st) {
  __shared__ int f;
  __syncthreads();
  if (threadIdx.x == 0) f = failed(st) ? 1 : 0;
  __syncthreads();
  return f != 0;
}

__device__ __forceinline__ bool warp_failed(const pwp_stats* st) {
  int f = 0;
  if ((threadIdx.x & 31) == 0) f = failed(st) ? 1 : 0;
  return __shfl_sync(0xffffffffu, f, 0) != 0;
}

__device__ __forceinline__ void set_error(pwp_stats* st, int status, int site) {
  if (atomicCAS((int*)&st->status, PWP_OK, status) == PWP_OK) st->status_site = site;
}

// Monotone key of a non-negative fp32 score: its bit pattern with the sign bit cleared
// (a NaN of either sign stays inside the 31-bit key range the histograms cover).
__device__ __forceinline__ unsigned int score_key(float s) { return __float_as_uint(s) & 0x7fffffffu; }

// Thanos ranks by |W| * ||X_q|| (Wanda score).
__device__ __forceinline__ float wanda_score(float w, float xnorm) { return fabsf(w) * xnorm; }

// SparseGPT ranks by W^2 / [H^-1]_qq = (W / U_qq)^2.
__device__ __forceinline__ float obs_score(float w, float uqq) {
  float t = w / uqq;
  return t * t;
}

enum ScoreKind { kNoScore = 0, kWanda = 1, kObs = 2 };

// Head of an fp32 value in TF32 (round to nearest, ties away from zero).  With
// lo = x - head (exact in fp32), x == head + lo; the tensor-core update multiplies
// head*head + head*lo + lo*head, which carries fp32-level accuracy.
__device__ __forceinline__ float tf32_head(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return __uint_as_float(r);
}

template <int SCORE>
__device__ __forceinline__ unsigned int key_of(float w, float p) {
  return SCORE == kWanda ? score_key(wanda_score(w, p)) : score_key(obs_score(w, p));
}

// Counter increments whose old value nobody reads: reductions (red), which the issuing
// thread does not wait for, unlike an atomic that returns the old value.
__device__ __forceinline__ void red_add_shared(unsigned int* p, unsigned int v) {
  asm volatile("red.shared.add.u32 [%0], %1;" ::"r"((unsigned int)__cvta_generic_to_shared(p)), "r"(v) : "memory");
}
__device__ __forceinline__ void red_add_global(unsigned int* p, unsigned int v) {
  asm volatile("red.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Level-2 histogram entry of a key whose level-1 bin is the predicted one (pred is
// 0xffffffff when there is no prediction): the exact count plus its 512-bin summary.
__device__ __forceinline__ void count_level2(unsigned int key, unsigned int pred, unsigned int* __restrict__ h2,
                                             unsigned int* __restrict__ h2s) {
  if ((key >> kKeyLoBits) == pred) {
    const unsigned int lo = key & (unsigned int)(kHist2Bins - 1);
    red_add_global(&h2[lo], 1u);
    red_add_global(&h2s[lo >> kHist2SumShift], 1u);
  }
}

// Selection flag of one entry of block row k (column qq of the block).
// Unstructured: key < T, or key == T with column-major position qq*c + k at or before
// the tie cut-off.  N:M: rank inside the group of nm_m lanes by (key, column) below
// nm_m - nm_n.  Every lane of the warp must call it (N:M shuffles within the group).
template <bool NM>
__device__ __forceinline__ bool selected(unsigned int key, bool valid, int qq, int k, int c,
                                         const Ctl& ctl, int nm_n, int nm_m) {
  if (NM) {
    const int lane = threadIdx.x & 31;
    const int base = lane & ~(nm_m - 1);
    int rank = 0;
    for (int o = 0; o < nm_m; ++o) {
      unsigned int ko = __shfl_sync(0xffffffffu, key, base + o);
      rank += (ko < key) || (ko == key && base + o < lane);
    }
    return valid && rank < nm_m - nm_n;
  }
  if (!valid || ctl.mode == 0) return false;
  if (key < ctl.T) return true;
  if (key == ctl.T) return (long long)qq * c + k <= ctl.pstar;
  return false;
}

// ---------------------------------------------------------------- instrumentation (host side)
enum KernelClass { kKHessian = 0, kKFactor = 1, kKStream = 2, kKSelect = 3, kKSolve = 4, kKRowPrune = 5,
                   kKColNorm = 6 };
void prof_begin(int which, cudaStream_t s);
void prof_end(int which, cudaStream_t s);
void count_launches(long long n);
// Polls every ordinary bounded device-side wait makes before giving up (pwp_set_wait_limit).
long long wait_limit();

// ---------------------------------------------------------------- launchers (host side)
cudaError_t launch_hessian(const void* X, int xtype, long long n, int b, float* H, int beta,
                           cudaStream_t s);
cudaError_t launch_damp_factor(float* H, int b, float damp, float* g_diag, void* ws,
                               size_t ws_bytes, pwp_stats* st, cudaStream_t s);
size_t factor_ws_bytes(int b);

// Level-2 histograms of one block: `pred` is filled by the scoring pass for the predicted
// level-1 bin, `reread` by the re-read when the prediction missed; each with its summary.
struct Level2 {
  unsigned int* pred;
  unsigned int* pred_sum;
  unsigned int* reread;
  unsigned int* reread_sum;
  unsigned int* tie_count;   // kMaxBlock per-column counts of entries tied at T
};

// The level-2 histograms a block's selection counted into (the control block's dirty
// flags, set when the level-1 bin is taken), cleared for the next block by the grid of the
// kernel that follows the selection (the row solve): thread gtid of stride.
__device__ __forceinline__ void clear_used_level2(const Ctl& ctl, Level2 l2, int gtid, int stride) {
  const uint4 z = make_uint4(0u, 0u, 0u, 0u);
  if (ctl.dirty_pred) {
    for (int i = gtid; i < kHist2Bins / 4; i += stride) reinterpret_cast<uint4*>(l2.pred)[i] = z;
    for (int i = gtid; i < kHist2SumBins / 4; i += stride) reinterpret_cast<uint4*>(l2.pred_sum)[i] = z;
  }
  if (ctl.dirty_reread) {
    for (int i = gtid; i < kHist2Bins / 4; i += stride) reinterpret_cast<uint4*>(l2.reread)[i] = z;
    for (int i = gtid; i < kHist2SumBins / 4; i += stride) reinterpret_cast<uint4*>(l2.reread_sum)[i] = z;
  }
}

// Selection arguments of the scoring pass that precedes a block's selection: the region's
// entry count and the budget (the residual global count, or the block quota); the pass's
// last CTA takes the level-1 bin and, when predicted, the exact threshold (pick.cuh).
struct PickArgs {
  long long region_n;
  long long quota;
  int global_budget;
  int enabled;
};

// The rest of the exact selection of a block (select.cu), two launches: the re-read when
// the level-1 bin was not predicted, then the cut-off among tied entries (each a no-op
// when not needed).
void launch_select_finish(int score, Ctl* ctl, Level2 l2, const float* W, int c, int b, int j, int j1, int q1,
                          const float* sc, pwp_stats* st, cudaStream_t s);
void launch_sweep_select(int step, int score, Ctl* ctl, unsigned int* hist1, Level2 l2, PickArgs pk, const float* W,
                         int c, int b, int j, int j1, int q1, const float* sc, const unsigned int* ties_all, int world,
                         int rank, pwp_stats* st, cudaStream_t s);

// W[:, u0:b] -= Z R on the tensor cores (stream_tc.cu), fused with zeroing the previous
// block's removals and the level-1 histogram of the scores of columns [j, hist_end).
// W is c x b with row stride ldw (mask: row stride b); with `upper` (c == b, u0 == 0)
// only the 128x128 tiles on or above the diagonal are visited.  Z (c x Bp, row stride ldz) and R,
// stored transposed (b x Bp, row stride ldz), come as TF32 head and fp32 remainder
// arrays.  Returns false, launching nothing, when the shape or alignment does not allow
// the tensor-core path.  spare_sms > 0 keeps that many SMs out of the persistent grid (for
// a kernel that runs beside it on another stream); keep >= 0 (score kNoScore; a multiple of
// 16) leaves the block [keep, keep + 64)^2 of W as it was.
bool launch_stream_tc(int score, float* W, int c, int b, int ldw, int u0, int j, const float* Zhi, const float* Zlo,
                      int Bp, int ldz, const float* Rhi, const float* Rlo, const uint8_t* mask, const float* sc,
                      int hist_end, unsigned int* hist1, Ctl* ctl, Level2 l2, pwp_stats* st,
                      cudaStream_t s, cudaError_t* err, bool upper = false, PickArgs pick = PickArgs{},
                      int spare_sms = 0, int keep = -1);

// Wanda / magnitude: per-row quota or N:M groups, no weight update (rowprune.cu).  H
// (its diagonal) or X ([n, b]) gives ||X_q|| for Wanda.
size_t no_update_ws_bytes(int b);
cudaError_t launch_no_update(const pwp_config* cfg, const void* W, int wtype, int c, int b, const float* H,
                             const void* X, int xtype, long long n, float* Wout, uint8_t* mask, void* ws,
                             pwp_stats* st, bool stats_ready, cudaStream_t s);

// the alpha variant (alpha.cu): outlier rows kept dense, the others pruned compactly
int alpha_rows(const pwp_config* cfg, int c);
size_t alpha_ws_bytes(size_t inner, int c, int b, int n_out);
cudaError_t launch_prune_alpha(const pwp_config* cfg, const void* W, int wtype, int c, int b, float* H, float* Wout,
                               uint8_t* mask, void* ws, size_t inner_bytes, pwp_stats* st, cudaStream_t s,
                               bool stats_ready, int n_out,
                               cudaError_t (*inner_prune)(const pwp_config*, const void*, int, int, int, float*,
                                                          float*, uint8_t*, void*, pwp_stats*, cudaStream_t, bool));

// compressed 2:4 storage (pack24.cu)
cudaError_t launch_pack24(const float* What, const uint8_t* mask, int c, int b, uint16_t* values, uint32_t* meta,
                          pwp_stats* st, cudaStream_t s);

// The prune's block loop with its finished column blocks of W-hat and the mask copied to
// pinned host memory as it goes (prune.cu; the host entry point in api.cu): each block's
// copies wait for an event recorded on the prune's stream and run on `copy`.
struct HostOut {
  float* W_host;
  uint8_t* mask_host;
  cudaStream_t copy;
  cudaEvent_t ev;
};
cudaError_t launch_prune_out(const pwp_config* cfg, const void* W, int wtype, int c, int b, float* H,
                             float* Wout, uint8_t* mask, void* ws, pwp_stats* st, cudaStream_t s,
                             bool stats_ready, const HostOut* ho);

// per-row work of one block (solve.cu); returns the number of kernels launched
// (both also clear the level-2 histograms the block's selection used)
int launch_thanos_solve(bool nm, const float* W, int c, int b, int j, int B, const float* Kt,
                        const float* xnorm, Ctl* ctl, Level2 l2, uint8_t* mask, float* Zs, int nm_n, int nm_m,
                        float* gscratch, pwp_stats* st, cudaStream_t s);
size_t solve_scratch_bytes(int c, int B, bool nm, int nm_n, int nm_m);
int launch_sparsegpt_solve(bool nm, const float* W, int c, int b, int j, int B, const float* H,
                           const float* udiag, Ctl* ctl, Level2 l2, uint8_t* mask, float* Zs, int nm_n,
                           int nm_m, pwp_stats* st, cudaStream_t s);

}  // namespace pwp
