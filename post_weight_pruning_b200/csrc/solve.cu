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

// Per warp: rows 0..NS-1 of the packed factor, the u/y vector and the selected indices in
// shared memory; rows NS..SCAP-1 (only rows with more than NS selections reach them) in a
// per-warp slot of global scratch.
template <int SCAP, int NS>
struct SolveSmem {
  static constexpr int kL = poff(NS);
  static constexpr int kY = SCAP + 4;
  static constexpr int kPerWarp = kL + kY + SCAP;  // floats: L, y, Qidx
  static constexpr int kGlobal = poff(SCAP) - poff(NS);   // floats of global scratch per warp
};

template <int NS>
struct Rows {
  float* L;   // shared, rows < NS
  float* G;   // global, rows >= NS
  __device__ __forceinline__ float* row(int i) const { return i < NS ? L + poff(i) : G + (poff(i) - poff(NS)); }
};

// Cholesky R-hat = L L^T (left-looking, 8-column panels; lanes own rows) with u carried
// as an extra row so that the factorisation also gives y = L^-1 u, then L^T z = y.
// L holds R-hat's lower triangle on entry; y holds u.  On return y[0..s) = z.
// Per panel [jp, jp+8), the rows i in [jp, s] (s: the u row) go over the lanes in rounds
// of 32: each takes the contributions of columns < jp (float4 dot products against the
// eight panel rows), then in the first round the 8x8 diagonal block, held by lanes
// 0..7, is factored with shuffles; every other row finishes its eight panel entries by
// forward substitution.  A packed row i holds columns up to 4*(i/4)+3, so rows jp..jp+3
// of a panel touch only its first four columns.  One __syncwarp per panel.  The
// reciprocal of every diagonal entry goes to idg for the back substitution.  Returns
// false on a non-positive pivot (uniform).
template <int SCAP, int NS>
__device__ bool chol_solve(const Rows<NS> R, float* __restrict__ y, float* __restrict__ idg, int s, int lane) {
  for (int jp = 0; jp < s; jp += 8) {
    const int pw = min(8, s - jp);
    const float* pr[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) pr[c] = R.row(jp + (c < pw ? c : 0));   // padding rows: any valid row
    const int nr = (s - jp + 1 + 31) >> 5;
    float Ld[8][8];
    float il[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      il[c] = 1.f;
#pragma unroll
      for (int c2 = 0; c2 < 8; ++c2) Ld[c][c2] = 0.f;
    }
    for (int r = 0; r < nr; ++r) {
      const int i = jp + lane + 32 * r;
      float* ri = (i < s) ? R.row(i) : y;
      const bool two = (i >= jp + 4) || (i >= s);   // the row holds panel columns jp+4..
      float acc[8];
      {
        const float4 a = *reinterpret_cast<const float4*>(ri + jp);
        acc[0] = a.x; acc[1] = a.y; acc[2] = a.z; acc[3] = a.w;
        float4 bq = make_float4(0.f, 0.f, 0.f, 0.f);
        if (two) bq = *reinterpret_cast<const float4*>(ri + jp + 4);
        acc[4] = bq.x; acc[5] = bq.y; acc[6] = bq.z; acc[7] = bq.w;
      }
#pragma unroll 2
      for (int t = 0; t < jp; t += 4) {
        const float4 x = *reinterpret_cast<const float4*>(ri + t);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const float4 q = *reinterpret_cast<const float4*>(pr[c] + t);
          float v = acc[c];
          v = fmaf(-x.x, q.x, v);
          v = fmaf(-x.y, q.y, v);
          v = fmaf(-x.z, q.z, v);
          v = fmaf(-x.w, q.w, v);
          acc[c] = v;
        }
      }
      if (r == 0) {
        // the 8x8 diagonal block: rows jp..jp+pw-1 are acc of lanes 0..pw-1
        bool ok = true;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          if (c < pw) {
            const float d = __shfl_sync(0xffffffffu, acc[c], c);
            if (!(d > 0.f)) { ok = false; break; }
            il[c] = rsqrtf(d);
            if (lane == c) acc[c] = d * il[c];
            else if (lane > c && lane < pw) acc[c] *= il[c];
            if (lane == 0) idg[jp + c] = il[c];
#pragma unroll
            for (int c2 = c + 1; c2 < 8; ++c2) {
              const float lc2 = __shfl_sync(0xffffffffu, acc[c], c2);   // L[jp+c2][jp+c]
              if (lane >= c2 && lane < pw) acc[c2] = fmaf(-acc[c], lc2, acc[c2]);
            }
          }
        }
        if (!ok) return false;
#pragma unroll
        for (int c = 0; c < 8; ++c)
#pragma unroll
          for (int c2 = 0; c2 <= c; ++c2) Ld[c][c2] = __shfl_sync(0xffffffffu, acc[c2], c);
      }
      if (i > s) continue;
      if (i < jp + pw && i < s) {
        *reinterpret_cast<float4*>(ri + jp) = make_float4(acc[0], acc[1], acc[2], acc[3]);
        if (two) *reinterpret_cast<float4*>(ri + jp + 4) = make_float4(acc[4], acc[5], acc[6], acc[7]);
      } else {
        float x[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          float v = acc[c];
#pragma unroll
          for (int c2 = 0; c2 < c; ++c2) v = fmaf(-x[c2], Ld[c][c2], v);
          x[c] = v * il[c];
        }
        *reinterpret_cast<float4*>(ri + jp) = make_float4(x[0], x[1], x[2], x[3]);
        *reinterpret_cast<float4*>(ri + jp + 4) = make_float4(x[4], x[5], x[6], x[7]);
      }
    }
    __syncwarp();
  }
  // back substitution L^T z = y, four rows at a time from the bottom: the 4x4 corner
  // is solved redundantly by every lane, then the rows above drop its contribution
  for (int a0 = (s - 1) & ~3; a0 >= 0; a0 -= 4) {
    const int pw = min(4, s - a0);
    const float* rr[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) rr[c] = R.row(a0 + (c < pw ? c : pw - 1));
    float z[4];
#pragma unroll
    for (int c = 3; c >= 0; --c) {
      z[c] = 0.f;
      if (c < pw) {
        float v = y[a0 + c];
#pragma unroll
        for (int c2 = c + 1; c2 < 4; ++c2)
          if (c2 < pw) v = fmaf(-rr[c2][a0 + c], z[c2], v);
        z[c] = v * idg[a0 + c];
      }
    }
    __syncwarp();
    for (int t = lane; t < a0; t += 32) {
      float v = y[t];
#pragma unroll
      for (int c = 0; c < 4; ++c)
        if (c < pw) v = fmaf(-rr[c][t], z[c], v);
      y[t] = v;
    }
    if (lane < pw) y[a0 + lane] = z[lane];
    __syncwarp();
  }
  return true;
}

// One warp per row over a persistent grid (each warp keeps one scratch slot).  SCAP
// bounds the selected set; rows beyond NS of a large set live in the warp's global slot.
template <int SCAP, int NS, bool NM>
__global__ void __launch_bounds__(256) thanos_solve_kernel(const float* __restrict__ W, int c, int b,
                                                           int j, int B, const float* __restrict__ Kt,
                                                           const float* __restrict__ xnorm,
                                                           Ctl* __restrict__ ctlp,
                                                           uint8_t* __restrict__ mask,
                                                           float* __restrict__ Zs, int nm_n, int nm_m,
                                                           float* __restrict__ gscratch, pwp_stats* st) {
  extern __shared__ __align__(16) float smem[];
  if (warp_failed(st)) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nwarps = blockDim.x >> 5;
  const int slot = blockIdx.x * nwarps + warp;
  float* L = smem + warp * SolveSmem<SCAP, NS>::kPerWarp;
  float* y = L + SolveSmem<SCAP, NS>::kL;
  int* Qidx = reinterpret_cast<int*>(y + SolveSmem<SCAP, NS>::kY);
  const Rows<NS> R{L, gscratch ? gscratch + (size_t)slot * SolveSmem<SCAP, NS>::kGlobal : nullptr};
  const Ctl ctl = *ctlp;
  const int nJ = min(B, b - j);
  constexpr int MAXI = kMaxBlock / 32;
  for (int k = slot; k < c; k += gridDim.x * nwarps) {
    const float* wrow = W + (long long)k * b + j;
    float w[MAXI];
    bool sel[MAXI];
    int pos[MAXI];
    int s = 0;
#pragma unroll
    for (int i = 0; i < MAXI; ++i) {
      const int qq = lane + 32 * i;
      const bool valid = qq < nJ;
      w[i] = valid ? wrow[qq] : 0.f;
      const unsigned int key = valid ? key_of<kWanda>(w[i], __ldg(xnorm + j + qq)) : 0xffffffffu;
      sel[i] = (32 * i < nJ) ? selected<NM>(key, valid, qq, k, c, ctl, nm_n, nm_m) : false;
      const unsigned int bal = __ballot_sync(0xffffffffu, sel[i]);
      pos[i] = s + __popc(bal & ((1u << lane) - 1u));
      s += __popc(bal);
    }
    if (s > SCAP || (s > NS && !R.G)) {   // excluded by the launcher's choice of SCAP / scratch
      if (lane == 0) set_error(st, PWP_EINVAL, kSiteSolve);
      continue;
    }
    uint8_t* mrow = mask + (long long)k * b + j;
#pragma unroll
    for (int i = 0; i < MAXI; ++i) {
      const int qq = lane + 32 * i;
      if (qq < nJ) mrow[qq] = sel[i] ? 1 : 0;
      if (sel[i]) {
        Qidx[pos[i]] = qq;
        y[pos[i]] = w[i];
      }
    }
    __syncwarp();
    bool ok = true;
    if (s > 0) {
      // R-hat = K[Q, Q], lower triangle: row a is K row q_a, loaded whole (lane l holds
      // columns 4l..4l+3), and entry (a, cc) is picked from lane q_cc / 4 by shuffles
      constexpr int CH = (SCAP + 31) / 32;
      int qv[CH];
#pragma unroll
      for (int ch = 0; ch < CH; ++ch) qv[ch] = (lane + 32 * ch < s) ? Qidx[lane + 32 * ch] : 0;
      const bool vec = (B & 3) == 0;
      const int c4 = 4 * lane;
      for (int a0 = 0; a0 < s; a0 += 4) {
        // four K rows in flight, then the picks from registers
        float4 kv[4];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const int a = a0 + r;
          const float* krow = Kt + (size_t)(a < s ? Qidx[a] : Qidx[0]) * B;
          if (vec && c4 + 3 < nJ) {
            kv[r] = __ldg(reinterpret_cast<const float4*>(krow + c4));
          } else {
            kv[r].x = c4 < nJ ? __ldg(krow + c4) : 0.f;
            kv[r].y = c4 + 1 < nJ ? __ldg(krow + c4 + 1) : 0.f;
            kv[r].z = c4 + 2 < nJ ? __ldg(krow + c4 + 2) : 0.f;
            kv[r].w = c4 + 3 < nJ ? __ldg(krow + c4 + 3) : 0.f;
          }
        }
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const int a = a0 + r;
          if (a >= s) break;
#pragma unroll
          for (int ch = 0; ch < CH; ++ch) {
            if (32 * ch > a) break;
            const int src = qv[ch] >> 2, comp = qv[ch] & 3;
            const float vx = __shfl_sync(0xffffffffu, kv[r].x, src);
            const float vy = __shfl_sync(0xffffffffu, kv[r].y, src);
            const float vz = __shfl_sync(0xffffffffu, kv[r].z, src);
            const float vw = __shfl_sync(0xffffffffu, kv[r].w, src);
            const float v = comp == 0 ? vx : comp == 1 ? vy : comp == 2 ? vz : vw;
            const int cc = lane + 32 * ch;
            if (cc <= a) R.row(a)[cc] = v;
          }
        }
      }
      __syncwarp();
      __syncwarp();  // the selected indices are spent: their slots hold 1 / L_ii from here on
      ok = chol_solve<SCAP, NS>(R, y, reinterpret_cast<float*>(Qidx), s, lane);
      if (!ok && lane == 0) set_error(st, PWP_ENOTSPD, kSiteSolve);
      if (lane == 0) atomicAdd((unsigned long long*)&ctlp->pruned, (unsigned long long)s);
    }
    float* zrow = Zs + (long long)k * B;
    float* zlo = zrow + (long long)c * B;
#pragma unroll
    for (int i = 0; i < MAXI; ++i) {
      const int qq = lane + 32 * i;
      if (qq < B) {
        const float z = (qq < nJ && sel[i] && ok) ? y[pos[i]] : 0.f;
        const float h = tf32_head(z);
        zrow[qq] = h;
        zlo[qq] = z - h;
      }
    }
    __syncwarp();
  }
}

// SparseGPT in-block sweep, one warp per row (no shared memory): for each block column
// q in order, e = W_q / U_qq on a selected entry (0 otherwise) and the later block
// columns of the row drop e * U[q, .].  Writes e (the row of E) and the mask.
template <bool NM>
__global__ void __launch_bounds__(256) sparsegpt_solve_kernel(const float* __restrict__ W, int c, int b,
                                                              int j, int B, const float* __restrict__ H,
                                                              const float* __restrict__ udiag,
                                                              Ctl* __restrict__ ctlp,
                                                              uint8_t* __restrict__ mask,
                                                              float* __restrict__ Zs, int nm_n, int nm_m,
                                                              pwp_stats* st) {
  if (warp_failed(st)) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int k = blockIdx.x * (blockDim.x >> 5) + warp;
  if (k >= c) return;
  const Ctl ctl = *ctlp;
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

template <int SCAP, int NS, bool NM>
void launch_thanos_variant(const float* W, int c, int b, int j, int B, const float* Kt, const float* xnorm,
                           Ctl* ctl, uint8_t* mask, float* Zs, int nm_n, int nm_m, float* gscratch,
                           pwp_stats* st, cudaStream_t s) {
  constexpr int warps = 8;
  const int smem = warps * SolveSmem<SCAP, NS>::kPerWarp * 4;
  static std::atomic<unsigned long long> attr_done{0};
  if (first_on_device(attr_done))
    cudaFuncSetAttribute(thanos_solve_kernel<SCAP, NS, NM>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  const int grid = min((c + warps - 1) / warps, kSolveCtas);
  thanos_solve_kernel<SCAP, NS, NM><<<grid, warps * 32, smem, s>>>(W, c, b, j, B, Kt, xnorm, ctl, mask, Zs, nm_n,
                                                                  nm_m, gscratch, st);
}

}  // namespace

size_t solve_scratch_bytes(int c, int B, bool nm, int nm_n, int nm_m) {
  const int smax = nm ? B / nm_m * (nm_m - nm_n) : B;
  if (smax <= 80) return 0;
  const int grid = min((c + 7) / 8, kSolveCtas);  // the launch's grid (8 warps per CTA)
  return (size_t)grid * 8 * SolveSmem<kMaxBlock, kSolveNS>::kGlobal * sizeof(float);
}

// A row's selected set is at most min(B, block width) (unstructured) or exactly
// B (m-n)/m (N:M).  8-warp CTAs keep up to 80 rows of each warp's factor in shared memory
// (two CTAs per SM); when a block can hold larger sets (capacity 128, whose larger u/index
// vectors leave room for 79 rows at two CTAs per SM), rows 79..127 of a large set go to
// the warp's slot of global scratch.
int launch_thanos_solve(bool nm, const float* W, int c, int b, int j, int B, const float* Kt,
                        const float* xnorm, Ctl* ctl, uint8_t* mask, float* Zs, int nm_n, int nm_m,
                        float* gscratch, pwp_stats* st, cudaStream_t s) {
  const int smax = nm ? B / nm_m * (nm_m - nm_n) : min(B, b - j);
  if (smax <= 80) {
    if (nm)
      launch_thanos_variant<80, 80, true>(W, c, b, j, B, Kt, xnorm, ctl, mask, Zs, nm_n, nm_m, nullptr, st, s);
    else
      launch_thanos_variant<80, 80, false>(W, c, b, j, B, Kt, xnorm, ctl, mask, Zs, nm_n, nm_m, nullptr, st, s);
  } else {
    if (nm)
      launch_thanos_variant<kMaxBlock, kSolveNS, true>(W, c, b, j, B, Kt, xnorm, ctl, mask, Zs, nm_n, nm_m,
                                                       gscratch, st, s);
    else
      launch_thanos_variant<kMaxBlock, kSolveNS, false>(W, c, b, j, B, Kt, xnorm, ctl, mask, Zs, nm_n, nm_m,
                                                        gscratch, st, s);
  }
  return 1;
}

int launch_sparsegpt_solve(bool nm, const float* W, int c, int b, int j, int B, const float* H,
                           const float* udiag, Ctl* ctl, uint8_t* mask, float* Zs, int nm_n, int nm_m,
                           pwp_stats* st, cudaStream_t s) {
  const int grid = (c + 7) / 8;
  if (nm)
    sparsegpt_solve_kernel<true><<<grid, 256, 0, s>>>(W, c, b, j, B, H, udiag, ctl, mask, Zs, nm_n, nm_m, st);
  else
    sparsegpt_solve_kernel<false><<<grid, 256, 0, s>>>(W, c, b, j, B, H, udiag, ctl, mask, Zs, nm_n, nm_m, st);
  return 1;
}

}  // namespace pwp
