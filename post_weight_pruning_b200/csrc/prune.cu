// Layer prune driver: setup, the per-block sweep, and the stream kernel that applies
// each block's compensation to the still-active columns while rescoring them.
//
// "Pruning LLMs with Thanos":
//   - section "Contribution one: solve a selected set directly": delta_k = -z_k^T K[Q, A]
//     with z_k = R-hat^-1 u, K the inverse Hessian of the active region A = [j, b);
//   - section "Contribution two: keep the budget global and the execution local": the
//     five steps (residual count, rescoring of the active region, candidate set,
//     intersection with the block, joint solve) are the per-block sequence below.
// "Weight Pruning in Large Language Models ..." (llms.blog), section "SparseGPT": the
// column update with the Cholesky factor of H^-1, applied block by block.
//
// With U upper and H_d^-1 = U^T U, the active inverse is K[J, A] = U[J,J]^T U[J, A] for
// the block J = [j, j+B) (the trailing principal inverse of an upper Cholesky factor
// is U[A,A]^T U[A,A]).  K_t = K[J_t, j_t:b] is formed once per block, so every row's
// update -- inside the block and beyond it -- is one product W[:, j:b] -= Z K_t with Z
// the rows' z scattered into B columns.  SparseGPT's sweep has the same shape with the
// rows of U in place of K_t.  That product is applied by the stream kernel of the next
// block, fused with rescoring the next active region and building its histogram.
#include "pick.cuh"

namespace pwp {

// ------------------------------------------------------------------ setup kernels

__global__ void init_stats_kernel(pwp_stats* st) {
  st->status = PWP_OK;
  st->status_site = 0;
  st->pruned = 0;
  st->target = 0;
  st->lambda = 0.f;
  st->shortfall = 0;
  st->reread_blocks = 0;
  st->tie_blocks = 0;
}

__global__ void init_ctl_kernel(Ctl* ctl, long long zstar, pwp_stats* st, long long target) {
  pdl_enter();
  ctl->zstar = zstar;
  ctl->pruned = 0;
  ctl->mode = 0;
  ctl->b1 = 0;
  ctl->b1_valid = 0;
  ctl->l2_ready = 0;
  ctl->dirty_pred = 0;
  ctl->dirty_reread = 0;
  ctl->tie_scan = 0;
  ctl->ticket = 0u;
  ctl->row_next = 0u;
  ctl->warps_done = 0u;
  st->target = target;
}

__global__ void convert_w_kernel(const void* __restrict__ W, int wtype, float* __restrict__ Wout,
                                 long long N) {
  pdl_enter();
  long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  long long stride = (long long)gridDim.x * blockDim.x;
  if (wtype == PWP_FP32) {
    const float* w = (const float*)W;
    for (; i < N; i += stride) Wout[i] = w[i];
  } else {
    const uint16_t* w = (const uint16_t*)W;
    for (; i < N; i += stride) Wout[i] = __uint_as_float(((unsigned int)w[i]) << 16);
  }
}

// ||X_q|| = sqrt(G_qq) for the Wanda score, U_qq for the OBS score.
__global__ void prep_diag_kernel(const float* __restrict__ H, int b, const float* __restrict__ g_diag,
                                 float* __restrict__ xnorm, float* __restrict__ udiag) {
  pdl_enter();
  int q = blockIdx.x * blockDim.x + threadIdx.x;
  if (q < b) {
    xnorm[q] = sqrtf(g_diag[q]);
    udiag[q] = H[(long long)q * b + q];
  }
}

// K_t[p][q] = sum_{r <= p} U[j+r][j+p] U[j+r][q] for p < |J_t|, q in [j_t, b): block t's
// rows of the active inverse.  Two forms: the in-block square K_t[:, j_t:j_t+B] in fp32
// (K_in, B x B per block, row stride B; the square is symmetric) for the row solves, and
// K_t transposed as TF32 head and fp32 remainder (K_hi, K_lo: b x B per block, row q
// holds column q of K_t, rows < j_t unused) -- the K-major operand of the tensor-core
// update.  Grid (column tiles of 128, blocks); 128 (p) x 128 (q) outputs per CTA, 8x8 per
// thread; the sum over r runs in chunks of 16 rows of U, double-buffered in shared memory
// (both operands are rows of U, read as float4; U's stale lower triangle is zeroed as it is
// loaded), and the tile is staged transposed, 64 columns at a time, so that every output
// row is written contiguously.
constexpr int kKmatChunk = 16;
__global__ void __launch_bounds__(256, 2) kmat_kernel(const float* __restrict__ H, int b, int B,
                                                   float* __restrict__ K_in, float* __restrict__ K_hi,
                                                   float* __restrict__ K_lo, const pwp_stats* st) {
  pdl_enter();
  __shared__ __align__(16) float sm[2 * 2 * kKmatChunk * 132];   // operands, then the staged tile
  float (*As)[kKmatChunk][132] = reinterpret_cast<float (*)[kKmatChunk][132]>(sm);
  float (*Bs)[kKmatChunk][132] = reinterpret_cast<float (*)[kKmatChunk][132]>(sm + 2 * kKmatChunk * 132);
  if (cta_failed(st)) return;
  const int t = blockIdx.y;
  const int j = t * B, nJ = min(B, b - j);
  const int q0 = j + blockIdx.x * 128;
  if (q0 >= b) return;
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  // loader: row r0 + (tid >> 5) + 8h of the chunk, columns 4 (tid & 31) .. + 3
  auto load = [&](int r0, float4 (&a)[2], float4 (&c)[2]) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int r = r0 + (tid >> 5) + 8 * h, col = 4 * (tid & 31);
      float va[4] = {0.f, 0.f, 0.f, 0.f}, vb[4] = {0.f, 0.f, 0.f, 0.f};
      if (r < nJ) {
        const float* urow = H + (long long)(j + r) * b;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int p = col + e, q = q0 + col + e;
          va[e] = (p < nJ && p >= r) ? urow[j + p] : 0.f;     // U[j+r][j+p], upper
          vb[e] = (q < b && q >= j + r) ? urow[q] : 0.f;      // U[j+r][q], upper
        }
      }
      a[h] = make_float4(va[0], va[1], va[2], va[3]);
      c[h] = make_float4(vb[0], vb[1], vb[2], vb[3]);
    }
  };
  float acc[8][8] = {};
  float4 ra[2], rb[2];
  int buf = 0;
  load(0, ra, rb);
  for (int r0 = 0; r0 < nJ; r0 += kKmatChunk) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int rr = (tid >> 5) + 8 * h, col = 4 * (tid & 31);
      *reinterpret_cast<float4*>(&As[buf][rr][col]) = ra[h];
      *reinterpret_cast<float4*>(&Bs[buf][rr][col]) = rb[h];
    }
    __syncthreads();
    if (r0 + kKmatChunk < nJ) load(r0 + kKmatChunk, ra, rb);
#pragma unroll
    for (int rr = 0; rr < kKmatChunk; ++rr) {
      const float4 a0 = *reinterpret_cast<const float4*>(&As[buf][rr][ty * 4]);
      const float4 a1 = *reinterpret_cast<const float4*>(&As[buf][rr][64 + ty * 4]);
      const float4 b0 = *reinterpret_cast<const float4*>(&Bs[buf][rr][tx * 4]);
      const float4 b1 = *reinterpret_cast<const float4*>(&Bs[buf][rr][64 + tx * 4]);
      const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int x = 0; x < 8; ++x)
#pragma unroll
        for (int y = 0; y < 8; ++y) acc[x][y] = fmaf(av[x], bv[y], acc[x][y]);
    }
    buf ^= 1;   // the next chunk goes to the other stage: one barrier per chunk suffices
  }
  // acc[x][y] = K_t[p][q] with p = (x < 4 ? 4ty + x : 64 + 4ty + x - 4), q = q0 + (same with tx, y)
  float* Kin = K_in + (size_t)t * B * B;
  float* Kh = K_hi + (size_t)t * b * B;
  float* Kl = K_lo + (size_t)t * b * B;
  float (*T)[129] = reinterpret_cast<float (*)[129]>(sm);   // 64 q rows x 128 p
  for (int half = 0; half < 2; ++half) {
    __syncthreads();   // the operands (or the previous half) are no longer read
#pragma unroll
    for (int y = 0; y < 8; ++y) {
      const int qq = y < 4 ? tx * 4 + y : 64 + tx * 4 + y - 4;
      if ((qq >> 6) != half) continue;
#pragma unroll
      for (int x = 0; x < 8; ++x) {
        const int p = x < 4 ? ty * 4 + x : 64 + ty * 4 + x - 4;
        T[qq & 63][p] = acc[x][y];
      }
    }
    __syncthreads();
    for (int idx = tid; idx < 64 * B; idx += blockDim.x) {
      const int qq = idx / B, p = idx - qq * B;
      const int q = q0 + half * 64 + qq;
      if (q >= b || p >= nJ) continue;
      const float v = T[qq][p];
      const float h = tf32_head(v);
      Kh[(size_t)q * B + p] = h;
      Kl[(size_t)q * B + p] = v - h;
      if (q < j + nJ) Kin[(size_t)(q - j) * B + p] = v;  // K_t[p][q] = K_t[q-j][j+p]
    }
  }
}


// ------------------------------------------------------------------ stream

// CUDA-core form of the update, for shapes the tensor-core kernel does not take.
// Over columns [u0, col_end):  W -= Z[:, 0:Bp] * R[0:Bp, :]  with Z = Zhi + Zlo and
// R = Rhi + Rlo (Rlo may be null; R row stride ldr, or stored transposed, R[k][q] at
// R[q*ldr + k], when r_trans; skipped when Bp == 0; with r_upper_from >= 0 the entries
// of R left of U's diagonal count as zero); entries of columns < j whose mask byte is set become exactly 0 (they
// are the previous block's removed weights, now final); for SCORE != 0 the top key bits
// (above kKeyLoBits) of every entry in columns [j, hist_end) go into the level-1 histogram.
// Tiles of 64 rows x 128 columns, persistent grid-stride loop.
template <int SCORE>
__global__ void __launch_bounds__(256) stream_kernel(float* __restrict__ W, int c, int b, int u0, int j,
                                                     int col_end, const float* __restrict__ Z,
                                                     const float* __restrict__ Zlo, int Bp, int ldz,
                                                     const float* __restrict__ R,
                                                     const float* __restrict__ Rlo, int ldr, int r_trans,
                                                     int r_upper_from, const uint8_t* __restrict__ mask,
                                                     const float* __restrict__ sc, int hist_end,
                                                     unsigned int* hist1, Ctl* ctl,
                                                     Level2 l2, PickArgs pk, pwp_stats* st) {
  pdl_enter();
  unsigned int* h2 = l2.pred;
  unsigned int* h2s = l2.pred_sum;
  __shared__ pick::Shared psh;
  extern __shared__ unsigned int shist[];  // kHist1Bins when SCORE != 0
  __shared__ float Zs[64][33];
  __shared__ __align__(16) float Rs[32][128];
  if (cta_failed(st)) return;
  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;
  if (SCORE != kNoScore)
    for (int i = tid; i < kHist1Bins; i += blockDim.x) shist[i] = 0u;
  const int ncols = col_end - u0;
  const int tiles_c = (ncols + 127) / 128, tiles_r = (c + 63) / 64;
  // level-1 bin of the previous block's threshold: its level-2 histogram is built here
  const unsigned int pred = (SCORE != kNoScore && ctl->b1_valid) ? ctl->b1 : 0xffffffffu;
  const long long ntiles = (long long)tiles_c * tiles_r;
  __syncthreads();
  for (long long tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
    const int r0 = (int)(tile / tiles_c) * 64;
    const int c0 = u0 + (int)(tile % tiles_c) * 128;
    float acc[4][8];
#pragma unroll
    for (int x = 0; x < 4; ++x)
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        int r = r0 + ty + 16 * x, q = c0 + tx + 16 * e;
        acc[x][e] = (r < c && q < col_end) ? W[(long long)r * b + q] : 0.f;
      }
    for (int k0 = 0; k0 < Bp; k0 += 32) {
      for (int idx = tid; idx < 64 * 32; idx += 256) {
        int rr = idx >> 5, kk = idx & 31;
        int r = r0 + rr, k = k0 + kk;
        Zs[rr][kk] = (r < c && k < Bp) ? Z[(long long)r * ldz + k] + Zlo[(long long)r * ldz + k] : 0.f;
      }
      for (int idx = tid; idx < 32 * 128; idx += 256) {
        int kk = idx >> 7, cc = idx & 127;
        int k = k0 + kk, q = c0 + cc;
        // r_upper_from >= 0: R's row k is row r_upper_from + k of the upper factor U, zero
        // left of the diagonal
        const bool in = k < Bp && q < col_end && (r_upper_from < 0 || q >= r_upper_from + k);
        const long long at = r_trans ? (long long)q * ldr + k : (long long)k * ldr + q;
        Rs[kk][cc] = in ? (Rlo ? R[at] + Rlo[at] : R[at]) : 0.f;
      }
      __syncthreads();
#pragma unroll 4
      for (int kk = 0; kk < 32; ++kk) {
        float zv[4], rv[8];
#pragma unroll
        for (int x = 0; x < 4; ++x) zv[x] = Zs[ty + 16 * x][kk];
#pragma unroll
        for (int e = 0; e < 8; ++e) rv[e] = Rs[kk][tx + 16 * e];
#pragma unroll
        for (int x = 0; x < 4; ++x)
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[x][e] = fmaf(-zv[x], rv[e], acc[x][e]);
      }
      __syncthreads();
    }
#pragma unroll
    for (int x = 0; x < 4; ++x) {
      const int r = r0 + ty + 16 * x;
      if (r >= c) continue;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const int q = c0 + tx + 16 * e;
        if (q >= col_end) continue;
        float v = acc[x][e];
        if (q < j) {
          if (mask[(long long)r * b + q]) v = 0.f;
          W[(long long)r * b + q] = v;
        } else {
          if (Bp > 0) W[(long long)r * b + q] = v;
          if (SCORE != kNoScore && q < hist_end) {
            unsigned int key = key_of<SCORE>(v, __ldg(sc + q));
            red_add_shared(&shist[key >> kKeyLoBits], 1u);
            count_level2(key, pred, h2, h2s);
          }
        }
      }
    }
  }
  if (SCORE != kNoScore) {
    __syncthreads();
    for (int i = tid; i < kHist1Bins; i += blockDim.x) {
      unsigned int v = shist[i];
      if (v) red_add_global(&hist1[i], v);
    }
    // the last CTA to finish takes the block's level-1 bin (and threshold, when predicted)
    if (pk.enabled) pick::after_scoring(ctl, hist1, l2, pk.region_n, pk.global_budget, pk.quota, st, psh);
  }
}

// Rows [jp, jp+Bp) of U over columns [jp, b), transposed (row q holds U[jp:jp+Bp, q],
// row stride B) as TF32 head and fp32 remainder, zero left of U's diagonal: SparseGPT's
// K-major operand of the tensor-core update.
__global__ void urows_kernel(const float* __restrict__ H, int b, int B, int jp, int Bp, float* __restrict__ Rhi,
                             float* __restrict__ Rlo, const pwp_stats* st) {
  pdl_enter();
  if (failed(st)) return;
  const long long n = (long long)Bp * (b - jp);
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
    const int k = (int)(i % Bp), q = jp + (int)(i / Bp);
    const float v = q >= jp + k ? H[(long long)(jp + k) * b + q] : 0.f;
    const float h = tf32_head(v);
    Rhi[(long long)q * B + k] = h;
    Rlo[(long long)q * B + k] = v - h;
  }
}

__global__ void finalize_kernel(const Ctl* ctl, pwp_stats* st, int check_budget) {
  pdl_enter();
  st->pruned = ctl->pruned;
  if (st->status == PWP_OK && check_budget && ctl->pruned != ctl->zstar)
    set_error(st, PWP_EBUDGET, kSiteFinal);
}

// ------------------------------------------------------------------ workspace

struct PruneBuffers {
  Ctl* ctl;
  unsigned int* hist1;
  Level2 l2;
  float* g_diag;
  float* xnorm;
  float* udiag;
  float* Zs;       // 2c x B: TF32 heads of Z, then the remainders
  float* K_in;     // Thanos: blocks x B x B, in-block inverse rows (fp32)
  float* K_hi;     // Thanos: blocks x b x B, inverse rows transposed, TF32 head
  float* K_lo;     //   ... and remainder
  float* R_hi;     // SparseGPT: b x B, the current block's rows of U transposed, TF32 head
  float* R_lo;     //   ... and remainder
  float* gscratch;
  void* fws;
  size_t fws_bytes;
};

static size_t align_up(size_t x) { return (x + 255) & ~(size_t)255; }

size_t prune_ws_layout(const pwp_config* cfg, int c, int b, PruneBuffers* pb, char* base) {
  if (cfg->method == PWP_WANDA || cfg->method == PWP_MAGNITUDE) return no_update_ws_bytes(b);
  const int n_out = alpha_rows(cfg, c);
  if (n_out > 0) {
    // the compact prune of the kept rows comes first (launch_prune lays it out itself)
    pwp_config ic = *cfg;
    ic.alpha = 0.f;
    return alpha_ws_bytes(prune_ws_layout(&ic, c - n_out, b, nullptr, nullptr), c, b, n_out);
  }
  const int B = cfg->block;
  const int nblk = (b + B - 1) / B;
  const bool thanos = cfg->method == PWP_THANOS;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off += align_up(bytes);
    return base ? (void*)(base + o) : nullptr;
  };
  PruneBuffers t;
  t.ctl = (Ctl*)take(sizeof(Ctl));
  t.hist1 = (unsigned int*)take(sizeof(unsigned int) * (kHist1Bins + 4));   // + a sweep's removal count
  // the level-2 arrays and the tie counts are contiguous, so one memset clears them
  t.l2.pred = (unsigned int*)take(sizeof(unsigned int) * (2 * kHist2Bins + 2 * kHist2SumBins + kMaxBlock));
  t.l2.pred_sum = t.l2.pred ? t.l2.pred + kHist2Bins : nullptr;
  t.l2.reread = t.l2.pred ? t.l2.pred_sum + kHist2SumBins : nullptr;
  t.l2.reread_sum = t.l2.pred ? t.l2.reread + kHist2Bins : nullptr;
  t.l2.tie_count = t.l2.pred ? t.l2.reread_sum + kHist2SumBins : nullptr;
  t.g_diag = (float*)take(sizeof(float) * b);
  t.xnorm = (float*)take(sizeof(float) * b);
  t.udiag = (float*)take(sizeof(float) * b);
  t.Zs = (float*)take(sizeof(float) * 2 * (size_t)c * B);
  t.K_in = thanos ? (float*)take(sizeof(float) * (size_t)nblk * B * B) : nullptr;
  t.K_hi = thanos ? (float*)take(sizeof(float) * (size_t)nblk * B * b) : nullptr;
  t.K_lo = thanos ? (float*)take(sizeof(float) * (size_t)nblk * B * b) : nullptr;
  t.R_hi = thanos ? nullptr : (float*)take(sizeof(float) * (size_t)B * b);
  t.R_lo = thanos ? nullptr : (float*)take(sizeof(float) * (size_t)B * b);
  const size_t gbytes = thanos ? solve_scratch_bytes(c, B, cfg->pattern == PWP_NM, cfg->nm_n, cfg->nm_m) : 0;
  t.gscratch = gbytes ? (float*)take(gbytes) : nullptr;
  t.fws_bytes = factor_ws_bytes(b);
  t.fws = take(t.fws_bytes);
  if (pb) *pb = t;
  return off;
}

// ------------------------------------------------------------------ driver

static std::atomic<int> g_nsm{0};
static std::atomic<unsigned long long> g_attr_done{0};

template <int SCORE>
static void launch_stream(float* W, int c, int b, int u0, int j, int col_end, const float* Z, const float* Zlo,
                          int Bp, int ldz, const float* R, const float* Rlo, int ldr, int r_trans, int r_upper_from,
                          const uint8_t* mask, const float* sc, int hist_end, unsigned int* hist1, Ctl* ctl,
                          Level2 l2, PickArgs pk, pwp_stats* st, cudaStream_t s) {
  const int smem = SCORE != kNoScore ? kHist1Bins * 4 : 0;
  const int tiles = ((col_end - u0 + 127) / 128) * ((c + 63) / 64);
  const int nsm = g_nsm.load();
  const int grid = tiles < nsm ? tiles : nsm;
  launch_pdl(stream_kernel<SCORE>, dim3(grid > 0 ? grid : 1), dim3(256), smem, s, W, c, b, u0, j, col_end, Z, Zlo, Bp, ldz, R, Rlo,
                                                             ldr, r_trans, r_upper_from, mask, sc, hist_end, hist1,
                                                             ctl, l2, pk, st);
}

static void launch_stream_any(int score, float* W, int c, int b, int u0, int j, const float* Z, const float* Zlo,
                              int Bp, int ldz, const float* R, const float* Rlo, int ldr, int r_trans,
                              int r_upper_from, const uint8_t* mask, const float* sc, int hist_end,
                              unsigned int* hist1, Ctl* ctl, Level2 l2, PickArgs pk, pwp_stats* st,
                              cudaStream_t s) {
  if (score == kWanda)
    launch_stream<kWanda>(W, c, b, u0, j, b, Z, Zlo, Bp, ldz, R, Rlo, ldr, r_trans, r_upper_from, mask, sc, hist_end,
                          hist1, ctl, l2, pk, st, s);
  else if (score == kObs)
    launch_stream<kObs>(W, c, b, u0, j, b, Z, Zlo, Bp, ldz, R, Rlo, ldr, r_trans, r_upper_from, mask, sc, hist_end,
                        hist1, ctl, l2, pk, st, s);
  else
    launch_stream<kNoScore>(W, c, b, u0, j, b, Z, Zlo, Bp, ldz, R, Rlo, ldr, r_trans, r_upper_from, mask, sc,
                            hist_end, hist1, ctl, l2, pk, st, s);
}

cudaError_t launch_stats_init(pwp_stats* st, cudaStream_t s) {
  init_stats_kernel<<<1, 1, 0, s>>>(st);
  count_launches(1);
  return cudaGetLastError();
}

// One prune's host-side state: the configuration, sizes, buffers and derived flags.
struct PruneRun {
  const pwp_config* cfg;
  int c, b, B, nblk;
  long long c_budget;   // rows the selection budget counts (c, or all ranks' rows for a sweep)
  bool thanos, nm, tc_shape;
  int score;
  float* H;
  float* Wout;
  uint8_t* mask;
  PruneBuffers pb;
  const float* sc;
  const float* Zlo;
  pwp_stats* st;
  cudaStream_t s;
};

static cudaError_t prune_init(PruneRun& R, const pwp_config* cfg, int c, int b, long long c_budget, float* H,
                              float* Wout, uint8_t* mask, void* ws, pwp_stats* st, cudaStream_t s) {
  R.cfg = cfg;
  R.c = c;
  R.b = b;
  R.B = cfg->block;
  R.nblk = (b + R.B - 1) / R.B;
  R.c_budget = c_budget;
  R.thanos = cfg->method == PWP_THANOS;
  R.nm = cfg->pattern == PWP_NM;
  R.score = R.nm ? kNoScore : (R.thanos ? kWanda : kObs);
  R.H = H;
  R.Wout = Wout;
  R.mask = mask;
  R.st = st;
  R.s = s;
  prune_ws_layout(cfg, c, b, &R.pb, (char*)ws);
  R.sc = R.thanos ? R.pb.xnorm : R.pb.udiag;
  R.Zlo = R.pb.Zs + (size_t)c * R.B;
  // tensor-core update: 16-byte rows for TMA (b, B multiples of 4), aligned W and mask
  R.tc_shape = (b % 4) == 0 && (R.B % 4) == 0 && ((uintptr_t)Wout % 16) == 0 && ((uintptr_t)mask % 4) == 0;
  if (first_on_device(g_attr_done)) {
    cudaError_t e0 = cudaFuncSetAttribute(stream_kernel<kWanda>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          kHist1Bins * 4);
    if (e0 == cudaSuccess)
      e0 = cudaFuncSetAttribute(stream_kernel<kObs>, cudaFuncAttributeMaxDynamicSharedMemorySize, kHist1Bins * 4);
    int dev = 0, nsm = kNumSM;
    if (e0 == cudaSuccess) e0 = cudaGetDevice(&dev);
    if (e0 == cudaSuccess) e0 = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
    if (e0 != cudaSuccess) {
      g_attr_done.fetch_and(~(1ull << (dev & 63)));   // try again on the next call
      return e0;
    }
    g_nsm = nsm;
  }
  return cudaSuccess;
}

// Removal target and budget of the layer (over c_budget rows).
static void prune_targets(const PruneRun& R, long long* zstar, long long* target) {
  const long long N = R.c_budget * R.b;
  *zstar = (long long)((double)R.cfg->sparsity * (double)N);
  if (R.nm) {
    *target = (long long)R.c * R.b / R.cfg->nm_m * (R.cfg->nm_m - R.cfg->nm_n);
  } else if (R.thanos) {
    *target = *zstar;
  } else {
    *target = 0;
    for (int t = 0; t < R.nblk; ++t)
      *target += (long long)((double)R.cfg->sparsity * (double)R.c_budget * (double)min(R.B, R.b - t * R.B));
  }
}

// Stats and control block, W-hat from W, the damped factor, the score scales and, for
// Thanos, every block's rows of the active inverse.
static cudaError_t prune_setup(PruneRun& R, const void* W, int wtype, bool stats_ready, long long* nl) {
  long long zstar, target;
  prune_targets(R, &zstar, &target);
  cudaStream_t s = R.s;
  if (!stats_ready) {
    init_stats_kernel<<<1, 1, 0, s>>>(R.st);
    ++*nl;
  }
  launch_pdl(init_ctl_kernel, dim3(1), dim3(1), 0, s, R.pb.ctl, zstar, R.st, target);
  cudaError_t em = cudaMemsetAsync(R.pb.hist1, 0, sizeof(unsigned int) * (kHist1Bins + 4), s);
  if (em == cudaSuccess)
    em = cudaMemsetAsync(R.pb.l2.pred, 0, sizeof(unsigned int) * (2 * kHist2Bins + 2 * kHist2SumBins + kMaxBlock),
                         s);
  if (em != cudaSuccess) return em;
  launch_pdl(convert_w_kernel, dim3(4 * g_nsm.load()), dim3(256), 0, s, W, wtype, R.Wout, (long long)R.c * R.b);
  *nl += 2;
  prof_begin(kKFactor, s);
  cudaError_t e = launch_damp_factor(R.H, R.b, R.cfg->damp, R.pb.g_diag, R.pb.fws, R.pb.fws_bytes, R.st, s);
  prof_end(kKFactor, s);
  if (e != cudaSuccess) return e;
  launch_pdl(prep_diag_kernel, dim3((R.b + 255) / 256), dim3(256), 0, s, (const float*)R.H, R.b,
             (const float*)R.pb.g_diag, R.pb.xnorm, R.pb.udiag);
  ++*nl;
  if (R.thanos) {
    dim3 g((R.b + 127) / 128, R.nblk);
    launch_pdl(kmat_kernel, dim3(g), dim3(256), 0, s, (const float*)R.H, R.b, R.B, R.pb.K_in,
               R.pb.K_hi, R.pb.K_lo, (const pwp_stats*)R.st);
    ++*nl;
  }
  return cudaGetLastError();
}

// Block t's selection arguments (t < nblk, scored patterns): the region's entry count and
// the budget, both over all c_budget rows.
static PickArgs pick_args(const PruneRun& R, int t, bool fused) {
  PickArgs pk{};
  if (R.score == kNoScore || t >= R.nblk) return pk;
  const int j = t * R.B, j1 = min(R.b, j + R.B);
  pk.region_n = R.thanos ? R.c_budget * (R.b - j) : R.c_budget * (j1 - j);
  pk.quota = R.thanos ? 0 : (long long)((double)R.cfg->sparsity * (double)R.c_budget * (double)(j1 - j));
  pk.global_budget = R.thanos ? 1 : 0;
  pk.enabled = fused ? 1 : 0;
  return pk;
}

// Pass t: apply block t-1's update to the active columns (t > 0) while scoring block t's
// region into the level-1 histogram (t < nblk); t = nblk only finishes the last block.
static cudaError_t prune_pass(PruneRun& R, int t, PickArgs pk, long long* nl) {
  const int b = R.b, B = R.B, c = R.c;
  const int j = t * B, j1 = min(b, j + B);
  const int jp = (t - 1) * B, Bp = t > 0 ? min(B, b - jp) : 0;
  const int u0 = t > 0 ? jp : j;
  const int jj = t == R.nblk ? b : j;
  const int pass_score = t == R.nblk ? kNoScore : R.score;
  const int hist_end = t == R.nblk ? b : (R.thanos ? b : j1);
  PruneBuffers& pb = R.pb;
  cudaStream_t s = R.s;
  prof_begin(kKStream, s);
  if (t > 0) {
    // W[:, jp:b] -= Z R with R = block t-1's rows of K (Thanos) or of U (SparseGPT)
    bool done = false;
    if (R.tc_shape) {
      const float* Rh = R.thanos ? pb.K_hi + (size_t)(t - 1) * b * B : pb.R_hi;
      const float* Rl = R.thanos ? pb.K_lo + (size_t)(t - 1) * b * B : pb.R_lo;
      if (!R.thanos) {
        const long long n = (long long)Bp * (b - jp);
        const int grid = (int)min((n + 255) / 256, (long long)8 * g_nsm.load());
        launch_pdl(urows_kernel, dim3(grid), dim3(256), 0, s, (const float*)R.H, b, B, jp, Bp, pb.R_hi, pb.R_lo,
                   (const pwp_stats*)R.st);
        ++*nl;
      }
      cudaError_t e2 = cudaSuccess;
      done = launch_stream_tc(pass_score, R.Wout, c, b, b, u0, jj, pb.Zs, R.Zlo, Bp, B, Rh, Rl, R.mask, R.sc,
                              hist_end, pb.hist1, pb.ctl, pb.l2, R.st, s, &e2, false, pk);
      if (e2 != cudaSuccess) return e2;
    }
    if (!done) {
      // Thanos: K_t transposed (row stride B); SparseGPT: U's rows in place in H
      const float* Rm = R.thanos ? pb.K_hi + (size_t)(t - 1) * b * B : R.H + (size_t)jp * b;
      const float* Rlo = R.thanos ? pb.K_lo + (size_t)(t - 1) * b * B : nullptr;
      launch_stream_any(pass_score, R.Wout, c, b, u0, jj, pb.Zs, R.Zlo, Bp, B, Rm, Rlo, R.thanos ? B : b,
                        R.thanos ? 1 : 0, R.thanos ? -1 : jp, R.mask, R.sc, hist_end, pb.hist1, pb.ctl, pb.l2, pk,
                        R.st, s);
    }
    ++*nl;
  } else if (R.score != kNoScore) {
    // first block: nothing to apply yet, only the scores of the active region
    launch_stream_any(R.score, R.Wout, c, b, j, j, pb.Zs, R.Zlo, 0, B, nullptr, nullptr, b, 0, -1, R.mask, R.sc,
                      hist_end, pb.hist1, pb.ctl, pb.l2, pk, R.st, s);
    ++*nl;
  }
  prof_end(kKStream, s);
  return cudaSuccess;
}

// Block t's per-row work: the masks, the joint solves (Thanos) or the column sweep
// (SparseGPT), and the rows' coefficients for the next pass.
static void prune_solve(PruneRun& R, int t, long long* nl) {
  const int j = t * R.B;
  prof_begin(kKSolve, R.s);
  if (R.thanos)
    *nl += launch_thanos_solve(R.nm, R.Wout, R.c, R.b, j, R.B, R.pb.K_in + (size_t)t * R.B * R.B, R.pb.xnorm,
                               R.pb.ctl, R.pb.l2, R.mask, R.pb.Zs, R.cfg->nm_n, R.cfg->nm_m, R.pb.gscratch, R.st, R.s);
  else
    *nl += launch_sparsegpt_solve(R.nm, R.Wout, R.c, R.b, j, R.B, R.H, R.pb.udiag, R.pb.ctl, R.pb.l2, R.mask, R.pb.Zs,
                                  R.cfg->nm_n, R.cfg->nm_m, R.st, R.s);
  prof_end(kKSolve, R.s);
}

// stats_ready: the caller already reset *st on this stream (and may have recorded an
// earlier device-side failure in it, which then turns this call's kernels into no-ops).
cudaError_t launch_prune(const pwp_config* cfg, const void* W, int wtype, int c, int b, float* H,
                         float* Wout, uint8_t* mask, void* ws, pwp_stats* st, cudaStream_t s,
                         bool stats_ready) {
  return launch_prune_out(cfg, W, wtype, c, b, H, Wout, mask, ws, st, s, stats_ready, nullptr);
}

// Block t-1's columns of W-hat and of the mask are final once pass t has run (it applies
// that block's update to columns >= jp and zeroes its removals; later passes start at
// column j_t): with `ho`, they go back to the host on its copy stream right then.
static void copy_block_out(const PruneRun& R, int tb, const HostOut* ho) {
  if (!ho || tb < 0 || tb >= R.nblk) return;
  const int jq = tb * R.B, w = min(R.B, R.b - jq);
  cudaEventRecord(ho->ev, R.s);
  cudaStreamWaitEvent(ho->copy, ho->ev, 0);
  cudaMemcpy2DAsync(ho->W_host + jq, (size_t)R.b * sizeof(float), R.Wout + jq, (size_t)R.b * sizeof(float),
                    (size_t)w * sizeof(float), (size_t)R.c, cudaMemcpyDeviceToHost, ho->copy);
  cudaMemcpy2DAsync(ho->mask_host + jq, (size_t)R.b, R.mask + jq, (size_t)R.b, (size_t)w, (size_t)R.c,
                    cudaMemcpyDeviceToHost, ho->copy);
}

cudaError_t launch_prune_out(const pwp_config* cfg, const void* W, int wtype, int c, int b, float* H,
                             float* Wout, uint8_t* mask, void* ws, pwp_stats* st, cudaStream_t s,
                             bool stats_ready, const HostOut* ho) {
  if (cfg->method == PWP_WANDA || cfg->method == PWP_MAGNITUDE)
    return launch_no_update(cfg, W, wtype, c, b, cfg->method == PWP_WANDA ? H : nullptr, nullptr, 0, 0, Wout,
                            mask, ws, st, stats_ready, s);
  const int n_out = alpha_rows(cfg, c);
  if (n_out > 0) {
    pwp_config ic = *cfg;
    ic.alpha = 0.f;
    const size_t inner = prune_ws_layout(&ic, c - n_out, b, nullptr, nullptr);
    return launch_prune_alpha(cfg, W, wtype, c, b, H, Wout, mask, ws, inner, st, s, stats_ready, n_out,
                              &launch_prune);
  }
  PruneRun R;
  cudaError_t e = prune_init(R, cfg, c, b, c, H, Wout, mask, ws, st, s);
  if (e != cudaSuccess) return e;
  long long nl = 0;
  e = prune_setup(R, W, wtype, stats_ready, &nl);
  if (e != cudaSuccess) return e;
  for (int t = 0; t <= R.nblk; ++t) {
    // block t's selection: the scoring pass's last CTA takes the level-1 bin (and the
    // threshold, when predicted); select_finish does the rest
    e = prune_pass(R, t, pick_args(R, t, true), &nl);
    if (e != cudaSuccess) return e;
    copy_block_out(R, t - 1, ho);
    if (t == R.nblk) break;
    if (R.score != kNoScore) {
      const int j = t * R.B, j1 = min(b, j + R.B);
      prof_begin(kKSelect, s);
      launch_select_finish(R.score, R.pb.ctl, R.pb.l2, Wout, c, b, j, j1, R.thanos ? b : j1, R.sc, st, s);
      prof_end(kKSelect, s);
      nl += 2;
    }
    prune_solve(R, t, &nl);
  }
  launch_pdl(finalize_kernel, dim3(1), dim3(1), 0, s, (const Ctl*)R.pb.ctl, st, (R.thanos && !R.nm) ? 1 : 0);
  count_launches(nl + 1);
  return cudaGetLastError();
}

// ---------------------------------------------------------------- the stepwise sweep
// The block loop of launch_prune taken apart, for rows sharded over ranks with the
// unstructured budget counted over every rank's rows (c_budget): the caller sums the
// level-1 histogram (with each rank's removal count), the level-2 histograms and gathers
// the tie counts over ranks between the steps (pwp_sweep_step in include/pwp.h).
cudaError_t sweep_step(const pwp_config* cfg, const void* W, int wtype, int c, int b, long long c_budget, float* H,
                       float* Wout, uint8_t* mask, void* ws, pwp_stats* st, const unsigned int* ties_all, int world,
                       int rank, cudaStream_t s, int step, int t) {
  PruneRun R;
  cudaError_t e = prune_init(R, cfg, c, b, c_budget, H, Wout, mask, ws, st, s);
  if (e != cudaSuccess) return e;
  long long nl = 0;
  const int j = t * R.B, j1 = min(b, j + R.B), q1 = R.thanos ? b : j1;
  switch (step) {
    case PWP_SWEEP_SETUP:
      e = prune_setup(R, W, wtype, false, &nl);
      break;
    case PWP_SWEEP_SCORE:
      e = prune_pass(R, t, pick_args(R, t, false), &nl);
      if (e == cudaSuccess && t < R.nblk) {
        launch_sweep_select(0, R.score, R.pb.ctl, R.pb.hist1, R.pb.l2, PickArgs{}, Wout, c, b, j, j1, q1, R.sc,
                            nullptr, world, rank, st, s);
        ++nl;
      }
      break;
    case PWP_SWEEP_PICK_BIN:
    case PWP_SWEEP_REREAD:
    case PWP_SWEEP_PICK_KEY:
    case PWP_SWEEP_COUNT_TIES:
    case PWP_SWEEP_CUT_TIES: {
      const int k = step == PWP_SWEEP_PICK_BIN ? 1 : step == PWP_SWEEP_REREAD ? 2 : step == PWP_SWEEP_PICK_KEY ? 3
                    : step == PWP_SWEEP_COUNT_TIES ? 4 : 5;
      prof_begin(kKSelect, s);
      launch_sweep_select(k, R.score, R.pb.ctl, R.pb.hist1, R.pb.l2, pick_args(R, t, false), Wout, c, b, j, j1, q1,
                          R.sc, ties_all, world, rank, st, s);
      prof_end(kKSelect, s);
      ++nl;
      break;
    }
    case PWP_SWEEP_SOLVE:   // (also clears the block's level-2 histograms)
      prune_solve(R, t, &nl);
      break;
    case PWP_SWEEP_FINISH:
      e = prune_pass(R, R.nblk, PickArgs{}, &nl);
      launch_pdl(finalize_kernel, dim3(1), dim3(1), 0, s, (const Ctl*)R.pb.ctl, st, 0);
      ++nl;
      break;
    default:
      return cudaErrorInvalidValue;
  }
  count_launches(nl);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// Device addresses of the buffers the caller exchanges between ranks.
void sweep_buffers(const pwp_config* cfg, int c, int b, void* ws, unsigned int** level1, long long* n1,
                   unsigned int** level2, long long* n2, unsigned int** ties, long long* nt) {
  PruneBuffers pb;
  prune_ws_layout(cfg, c, b, &pb, (char*)ws);
  *level1 = pb.hist1;
  *n1 = kHist1Bins + 1;                          // + this rank's removal count
  *level2 = pb.l2.pred;
  *n2 = 2 * ((long long)kHist2Bins + kHist2SumBins);   // predicted and re-read, with their summaries
  *ties = pb.l2.tie_count;
  *nt = kMaxBlock;
}

}  // namespace pwp
