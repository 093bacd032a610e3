// The per-block compensation W[:, u0:b] -= Z R on the 5th-generation tensor cores,
// fused with finishing the previous block's removals and rescoring the active region.
//
// "Pruning LLMs with Thanos", section "Contribution one: solve a selected set directly":
// every row's update delta_k = -z_k^T K[Q, A] is a row of the product Z K_t (Z the z's
// scattered into the block's B columns); section "Contribution two: keep the budget
// global and the execution local", step 2: the active region is rescored on the updated
// weights before the next candidate set is formed.  For SparseGPT ("Weight Pruning in
// Large Language Models ...", section "SparseGPT") R is the block's rows of U.
//
// The product is a dense c x (b-u0) x B contraction.  It runs as TF32 MMAs with fp32
// accumulation in tensor memory; each operand comes as a TF32 head and its fp32
// remainder (x = head + lo), and the accumulator takes head*head + head*lo + lo*head,
// which keeps the product at fp32-level accuracy (the dropped lo*lo term is below 2^-22
// of it).  Both operands are K-major: Z is c x B (row stride B) and R is stored
// transposed, b x B (row q holds column q of R; TF32 operands stored N-major would need
// a different shared-memory atom than the plain 128-byte swizzle).
//
// One persistent CTA per SM walks 128 x 128 output tiles with four roles:
//   - warp 8 (one thread) streams 32-deep K slices of 128 rows of Z and of R^T with TMA
//     into a 2-stage ring, 128-byte swizzle;
//   - warp 9 (one thread) issues tcgen05.mma kind::tf32 (M 128, N 128, K 8) into one of
//     two 128-column accumulators, so the epilogue of one tile overlaps the MMAs of the
//     next;
//   - warp 10 (one thread) brings the tile of W into shared memory with TMA, in two
//     64-column halves with a buffer each, so a half loads while the other is worked on;
//   - warps 0-7 (warp w: tile rows 32(w%4).., columns 32(w/4).. of each half) read the
//     accumulator, subtract it from W in shared memory, set the previous block's removed
//     weights to exactly 0, histogram the score keys of columns [j, hist_end) in shared
//     memory (flushed to the level-1 histogram once per CTA), and one thread stores the
//     half back with TMA.
// Every wait is bounded; a wait that runs out records PWP_ETIMEOUT, the other roles stop
// at their next wait, and the epilogue warps take each stop decision together through a
// reducing barrier.  Copies and MMAs already in flight are always waited for before the
// CTA leaves.
#include "pick.cuh"
#include "tc_common.cuh"

namespace pwp {
namespace {

using namespace tc;

constexpr int TM = 128, TN = 128, TK = 32, STAGES = 2;
constexpr int A_BYTES = TM * TK * 4;                     // 16 KB: 128 rows x 128 bytes
constexpr int B_BYTES = TN * TK * 4;                     // 16 KB: 128 rows x 128 bytes
constexpr int STAGE_BYTES = 2 * A_BYTES + 2 * B_BYTES;   // heads and remainders of both
constexpr int W_BOX = TM * 32 * 4;                       // 16 KB: 128 rows x 32 columns of W (a quarter)
constexpr int kWBufs = 4;                                // the ring of W quarters
constexpr int W_OFF = STAGES * STAGE_BYTES;
constexpr int HIST_OFF = W_OFF + kWBufs * W_BOX;
constexpr int BAR_OFF = HIST_OFF + kHist1Bins * 4;
constexpr int SMEM_BYTES = 1024 + BAR_OFF + 256;
constexpr int kAccCols = 2 * TN;
constexpr int kEpiWarps = 8, kProducerWarp = 8, kMmaWarp = 9, kWLoadWarp = 10, kThreads = 352;
constexpr int kEpiBarrier = 1;
// kind::tf32 instruction descriptor: D fp32, A and B tf32, both K-major, N = 128, M = 128
constexpr uint32_t IDESC = (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)(TN >> 3) << 17) |
                           ((uint32_t)(TM >> 4) << 24);

static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");

__device__ __forceinline__ void mma_tf32(uint32_t tmem_d, uint64_t da, uint64_t db, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(da), "l"(db), "r"(IDESC), "r"(acc)
      : "memory");
}

// Origin of tile `tile` of the walk: every (m, n) tile, m fastest, or with `upper` (a
// square W, u0 = 0) only the tiles with m <= n, column by column.
__device__ __forceinline__ void tile_origin(int tile, int mt, int u0, int upper, int& m0, int& n0) {
  if (!upper) {
    m0 = (tile % mt) * TM;
    n0 = u0 + (tile / mt) * TN;
    return;
  }
  int n = (int)((sqrtf(8.f * (float)tile + 1.f) - 1.f) * 0.5f);
  while ((n + 1) * (n + 2) / 2 <= tile) ++n;
  while (n > 0 && n * (n + 1) / 2 > tile) --n;
  m0 = (tile - n * (n + 1) / 2) * TM;
  n0 = n * TN;
}

// Byte offset of the 16-byte unit u (columns 4u..4u+3) of row r in a 128-byte-swizzled box.
__device__ __forceinline__ uint32_t sw_off(int r, int u) { return (uint32_t)(r * 128 + ((u ^ (r & 7)) << 4)); }

template <int SCORE>
__global__ void __launch_bounds__(kThreads, 1)
    stream_tc_kernel(const __grid_constant__ CUtensorMap mzh, const __grid_constant__ CUtensorMap mzl,
                     const __grid_constant__ CUtensorMap mrh, const __grid_constant__ CUtensorMap mrl,
                     const __grid_constant__ CUtensorMap mw, int c, int b, int u0, int j, int Bp, int upper,
                     const uint8_t* __restrict__ mask, const float* __restrict__ sc, int hist_end,
                     unsigned int* hist1, Ctl* ctl, Level2 l2, PickArgs pk,
                     pwp_stats* st, long long spin, int keep) {
  unsigned int* h2 = l2.pred;
  unsigned int* h2s = l2.pred_sum;
  __shared__ pick::Shared psh;
  // the set-up below touches only this CTA's shared and tensor memory, so it runs before the
  // wait for the previous kernel (no kernel that can share an SM with this one holds tensor
  // memory: this one's shared memory leaves no room for another tensor-core CTA)
  pdl_release();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint8_t* wbuf = smem + W_OFF;
  unsigned int* shist = reinterpret_cast<unsigned int*>(smem + HIST_OFF);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + BAR_OFF);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;   // accumulator a holds a finished tile
  uint64_t* tempty = tfull + 2;       // accumulator a has been read out
  uint64_t* wfull = tempty + 2;       // W quarter buffer in shared memory
  uint64_t* wdone = wfull + kWBufs;   // W quarter buffer computed, to be stored
  uint64_t* drain = wdone + kWBufs;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;
  volatile int* abortp = &abort_flag;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int mt = (c + TM - 1) / TM;
  const int ntiles = upper ? mt * (mt + 1) / 2 : mt * ((b - u0 + TN - 1) / TN);
  const int nkc = (Bp + TK - 1) / TK;

  if (SCORE != kNoScore)
    for (int i = tid; i < kHist1Bins; i += kThreads) shist[i] = 0u;
  if (tid == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], kEpiWarps);
    }
    for (int q = 0; q < kWBufs; ++q) {
      mbar_init(&wfull[q], 1);
      mbar_init(&wdone[q], 1);
    }
    mbar_init(drain, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    abort_flag = 0;
  }
  if (warp == kMmaWarp) tmem_alloc(&tmem_slot, kAccCols);
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tmem = tmem_slot;
  pdl_wait();   // the previous kernel has completed and its writes are visible
  if (cta_failed(st)) {
    // leave as a whole CTA, the tensor memory given back
    if (warp == kMmaWarp) tmem_free(tmem, kAccCols);
    return;
  }
  // level-1 bin of the previous block's threshold: its level-2 histogram is built here
  const unsigned int pred = (SCORE != kNoScore && ctl->b1_valid) ? ctl->b1 : 0xffffffffu;

  if (warp == kProducerWarp) {
    if (lane == 0) {
      prefetch_map(&mzh);
      prefetch_map(&mzl);
      prefetch_map(&mrh);
      prefetch_map(&mrl);
      int it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
        int m0, n0;
        tile_origin(tile, mt, u0, upper, m0, n0);
        for (int kc = 0; kc < nkc; ++kc) {
          const int s = it % STAGES;
          if (it >= STAGES && !mbar_wait(&empty[s], ((it / STAGES) - 1) & 1, abortp, spin)) {
            ok = false;
            break;
          }
          mbar_expect_tx(&full[s], STAGE_BYTES);
          uint8_t* a = smem + s * STAGE_BYTES;
          tma_load_2d(a, &mzh, &full[s], kc * TK, m0);
          tma_load_2d(a + A_BYTES, &mzl, &full[s], kc * TK, m0);
          tma_load_2d(a + 2 * A_BYTES, &mrh, &full[s], kc * TK, n0);
          tma_load_2d(a + 2 * A_BYTES + B_BYTES, &mrl, &full[s], kc * TK, n0);
          ++it;
        }
      }
      if (!ok) *abortp = 1;
      // every copy issued lands before the CTA leaves (already true unless a role gave up)
      for (int k = it - STAGES > 0 ? it - STAGES : 0; k < it; ++k)
        mbar_wait(&full[k % STAGES], (k / STAGES) & 1, kDrainLimit);
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    if (lane == 0) {
      const uint32_t sbase = smem_u32(smem);
      int it = 0, tc = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x, ++tc) {
        const int acc = tc & 1;
        if (tc >= 2 && !mbar_wait(&tempty[acc], ((tc >> 1) - 1) & 1, abortp, spin)) {
          ok = false;
          break;
        }
        fence_after();
        const uint32_t d = tmem + (uint32_t)(acc * TN);
        for (int kc = 0; kc < nkc; ++kc) {
          const int s = it % STAGES;
          if (!mbar_wait(&full[s], (it / STAGES) & 1, abortp, spin)) {
            ok = false;
            break;
          }
          fence_after();
          const uint32_t ah = sbase + s * STAGE_BYTES, al = ah + A_BYTES;
          const uint32_t bh = ah + 2 * A_BYTES, bl = bh + B_BYTES;
#pragma unroll
          for (int kk = 0; kk < TK / 8; ++kk) {
            // K-major: a K step of 8 is 32 bytes inside each 128-byte row
            const uint64_t dah = sw128_desc(ah + kk * 32, 16, 1024);
            const uint64_t dal = sw128_desc(al + kk * 32, 16, 1024);
            const uint64_t dbh = sw128_desc(bh + kk * 32, 16, 1024);
            const uint64_t dbl = sw128_desc(bl + kk * 32, 16, 1024);
            mma_tf32(d, dah, dbh, (kc | kk) != 0 ? 1u : 0u);
            mma_tf32(d, dah, dbl, 1u);
            mma_tf32(d, dal, dbh, 1u);
          }
          mma_commit(&empty[s]);
          ++it;
        }
        if (!ok) break;
        mma_commit(&tfull[acc]);
      }
      if (!ok) *abortp = 1;
      mma_commit(drain);  // completes once every MMA issued so far has finished
      mbar_wait(drain, 0, kDrainLimit);
    }
    __syncwarp();
  } else if (warp == kWLoadWarp) {
    if (lane == 0) {
      // quarters g = 0, 1, .. of this CTA's walk (tile g/4, columns n0 + 32(g%4)..) in a
      // ring of kWBufs buffers: quarter g loads into the buffer of quarter g - kWBufs once
      // that one has been computed (wdone), stored, and read out of shared memory by its store
      prefetch_map(&mw);
      int issued = 0, stored = 0;
      bool ok = true;
      auto store_quarter = [&](int gs) -> bool {
        const int buf = gs % kWBufs;
        if (!mbar_wait(&wdone[buf], (gs / kWBufs) & 1, abortp, spin)) return false;
        int m0, n0;
        tile_origin(blockIdx.x + (gs >> 2) * gridDim.x, mt, u0, upper, m0, n0);
        // rows and columns outside W are not written
        tma_store_2d(&mw, wbuf + buf * W_BOX, n0 + 32 * (gs & 3), m0);
        bulk_commit();
        return true;
      };
      for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
        int m0, n0;
        tile_origin(tile, mt, u0, upper, m0, n0);
        for (int qt = 0; qt < 4; ++qt) {
          const int buf = issued % kWBufs;
          if (issued >= kWBufs) {
            if (!store_quarter(issued - kWBufs)) {
              ok = false;
              break;
            }
            ++stored;
            bulk_wait_read0();   // that store has read the buffer
          }
          mbar_expect_tx(&wfull[buf], W_BOX);
          tma_load_2d(wbuf + buf * W_BOX, &mw, &wfull[buf], n0 + 32 * qt, m0);
          ++issued;
        }
      }
      // the last quarters go back once computed (unless a role gave up)
      while (ok && stored < issued) {
        if (!store_quarter(stored)) {
          ok = false;
          break;
        }
        ++stored;
      }
      if (!ok) *abortp = 1;
      bulk_wait0();   // every store issued has completed
      // the last loads of W land before the CTA leaves, whether or not they were used
      for (int k = issued - kWBufs > 0 ? issued - kWBufs : 0; k < issued; ++k)
        mbar_wait(&wfull[k % kWBufs], (k / kWBufs) & 1, kDrainLimit);
    }
    __syncwarp();
  } else {
    // epilogue: warp w reads accumulator lanes 32(w%4).. (tile rows) and, in each W
    // quarter, the 16 columns 16(w/4)..; quarter g of the walk sits in buffer g % kWBufs
    const int quarter = warp & 3, colsel = warp >> 2;
    const int rl = quarter * 32 + lane;  // tile row of this thread
    int tc = 0, g = 0;
    bool stop = false;
    for (int tile = blockIdx.x; tile < ntiles && !stop; tile += gridDim.x, ++tc) {
      const int acc = tc & 1;
      int m0, n0;
      tile_origin(tile, mt, u0, upper, m0, n0);
      const int r = m0 + rl;
      const bool row_ok = r < c;
      bool ok = mbar_wait(&tfull[acc], (tc >> 1) & 1, abortp, spin);
      for (int qt = 0; qt < 4; ++qt, ++g) {
        const int buf = g % kWBufs;
        ok = ok && mbar_wait(&wfull[buf], (g / kWBufs) & 1, abortp, spin);
        ok = __all_sync(0xffffffffu, ok);
        if (ok) {
          fence_after();
          float v[16];
          tmem_ld16(tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * TN + qt * 32 + colsel * 16), v);
          if (qt == 3) {  // this warp is done with the accumulator
            fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[acc]);
          }
          const int q0 = n0 + qt * 32 + colsel * 16;
          uint8_t* box = wbuf + buf * W_BOX;
          if (SCORE == kNoScore && keep >= 0 && r >= keep && r < keep + 64 && q0 >= keep && q0 < keep + 64) {
            // the block [keep, keep + 64)^2 keeps its values (its 16-column groups lie wholly
            // inside or outside it: keep and q0 are multiples of 16)
#pragma unroll
            for (int e = 0; e < 16; ++e) v[e] = 0.f;
          }
          if (q0 + 16 <= j) {
            // previous block: apply, and zero the removed weights
            const uint32_t* mr = reinterpret_cast<const uint32_t*>(mask + (long long)r * b + q0);
#pragma unroll
            for (int uu = 0; uu < 4; ++uu) {
              float4* p4 = reinterpret_cast<float4*>(box + sw_off(rl, 4 * colsel + uu));
              float4 w4 = *p4;
              const uint32_t mb = row_ok ? mr[uu] : 0u;
              w4.x = (mb & 0xffu) ? 0.f : w4.x - v[4 * uu];
              w4.y = (mb & 0xff00u) ? 0.f : w4.y - v[4 * uu + 1];
              w4.z = (mb & 0xff0000u) ? 0.f : w4.z - v[4 * uu + 2];
              w4.w = (mb & 0xff000000u) ? 0.f : w4.w - v[4 * uu + 3];
              *p4 = w4;
            }
          } else if (q0 >= j && q0 + 16 <= hist_end && q0 + 16 <= b) {
            // active columns, all scored
            float4 s4[4];
            if (SCORE != kNoScore) {
#pragma unroll
              for (int uu = 0; uu < 4; ++uu) s4[uu] = __ldg(reinterpret_cast<const float4*>(sc + q0 + 4 * uu));
            }
#pragma unroll
            for (int uu = 0; uu < 4; ++uu) {
              float4* p4 = reinterpret_cast<float4*>(box + sw_off(rl, 4 * colsel + uu));
              float4 w4 = *p4;
              w4.x -= v[4 * uu];
              w4.y -= v[4 * uu + 1];
              w4.z -= v[4 * uu + 2];
              w4.w -= v[4 * uu + 3];
              *p4 = w4;
              if (SCORE != kNoScore && row_ok) {
                const unsigned int k0 = key_of<SCORE>(w4.x, s4[uu].x), k1 = key_of<SCORE>(w4.y, s4[uu].y);
                const unsigned int k2 = key_of<SCORE>(w4.z, s4[uu].z), k3 = key_of<SCORE>(w4.w, s4[uu].w);
                red_add_shared(&shist[k0 >> kKeyLoBits], 1u);
                red_add_shared(&shist[k1 >> kKeyLoBits], 1u);
                red_add_shared(&shist[k2 >> kKeyLoBits], 1u);
                red_add_shared(&shist[k3 >> kKeyLoBits], 1u);
                count_level2(k0, pred, h2, h2s);
                count_level2(k1, pred, h2, h2s);
                count_level2(k2, pred, h2, h2s);
                count_level2(k3, pred, h2, h2s);
              }
            }
          } else if (q0 < b) {
            // mixed chunk (block edge, scored-range edge or the layer's last columns)
#pragma unroll
            for (int uu = 0; uu < 4; ++uu) {
              float4* p4 = reinterpret_cast<float4*>(box + sw_off(rl, 4 * colsel + uu));
              float o[4];
              {
                const float4 w4 = *p4;
                o[0] = w4.x - v[4 * uu];
                o[1] = w4.y - v[4 * uu + 1];
                o[2] = w4.z - v[4 * uu + 2];
                o[3] = w4.w - v[4 * uu + 3];
              }
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const int q = q0 + 4 * uu + e;
                if (!row_ok || q >= b) continue;
                if (q < j) {
                  if (mask[(long long)r * b + q]) o[e] = 0.f;
                } else if (SCORE != kNoScore && q < hist_end) {
                  const unsigned int key = key_of<SCORE>(o[e], __ldg(sc + q));
                  red_add_shared(&shist[key >> kKeyLoBits], 1u);
                  count_level2(key, pred, h2, h2s);
                }
              }
              *p4 = make_float4(o[0], o[1], o[2], o[3]);
            }
          }
          fence_proxy_async_smem();
        }
        stop = barrier_or(kEpiBarrier, kEpiWarps * 32, !ok || *abortp);
        if (stop) break;
        if (tid == 0) mbar_arrive(&wdone[buf]);   // the quarter is computed: the W thread stores it
      }
      if (stop && lane == 0) *abortp = 1;
    }
  }

  fence_before();
  __syncthreads();
  fence_after();
  if (warp == kMmaWarp) tmem_free(tmem, kAccCols);
  if (tid == 0 && *abortp) set_error(st, PWP_ETIMEOUT, kSiteStream);
  if (SCORE != kNoScore) {
    for (int i = tid; i < kHist1Bins; i += kThreads) {
      const unsigned int v = shist[i];
      if (v) red_add_global(&hist1[i], v);
    }
    // the last CTA to finish takes the block's level-1 bin (and threshold, when predicted)
    if (pk.enabled) pick::after_scoring(ctl, hist1, l2, pk.region_n, pk.global_budget, pk.quota, st, psh, shist);
  }
}

template <int SCORE>
cudaError_t launch_variant(const CUtensorMap* maps, int c, int b, int u0, int j, int Bp, int upper,
                           const uint8_t* mask, const float* sc, int hist_end, unsigned int* hist1, Ctl* ctl,
                           Level2 l2, PickArgs pk, pwp_stats* st, cudaStream_t s, int spare_sms, int keep) {
  static std::atomic<unsigned long long> attr_done{0};
  if (first_on_device(attr_done)) {
    cudaError_t e = cudaFuncSetAttribute(stream_tc_kernel<SCORE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         SMEM_BYTES);
    if (e != cudaSuccess) return e;
  }
  int dev = 0, nsm = kNumSM;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  const int mt = (c + TM - 1) / TM;
  const int ntiles = upper ? mt * (mt + 1) / 2 : mt * ((b - u0 + TN - 1) / TN);
  nsm = nsm - spare_sms > 1 ? nsm - spare_sms : 1;
  const int grid = ntiles < nsm ? ntiles : nsm;
  launch_pdl(stream_tc_kernel<SCORE>, dim3(grid), dim3(kThreads), SMEM_BYTES, s, maps[0], maps[1], maps[2], maps[3],
             maps[4], c, b, u0, j, Bp, upper, mask, sc, hist_end, hist1, ctl, l2, pk, st, wait_limit(), keep);
  return cudaGetLastError();
}

// fp32 2-D tensor map: `inner` contiguous elements per row, `rows` rows `ld` apart,
// boxes of box_x x box_y, 128-byte swizzle, zero fill outside.
bool encode_f32(CUtensorMap* map, const float* base, int inner, int rows, int ld, int box_x, int box_y) {
  PFN_cuTensorMapEncodeTiled_v12000 encode = tensor_map_encoder();
  if (!encode) return false;
  cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)ld * 4};
  cuuint32_t box[2] = {(cuuint32_t)box_x, (cuuint32_t)box_y};
  cuuint32_t estr[2] = {1, 1};
  return encode(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(base), dims, strides, box, estr,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool launch_stream_tc(int score, float* W, int c, int b, int ldw, int u0, int j, const float* Zhi, const float* Zlo,
                      int Bp, int ldz, const float* Rhi, const float* Rlo, const uint8_t* mask, const float* sc,
                      int hist_end, unsigned int* hist1, Ctl* ctl, Level2 l2, pwp_stats* st, cudaStream_t s,
                      cudaError_t* err, bool upper, PickArgs pk, int spare_sms, int keep) {
  *err = cudaSuccess;
  if (upper && (c != b || u0 != 0)) return false;
  // b, u0 multiples of 4: the epilogue moves whole float4s of W and 4-byte words of mask
  if (c < 1 || Bp < 1 || Bp > ldz || u0 >= b || (b % 4) != 0 || (ldw % 4) != 0 || ldw < b || (ldz % 4) != 0 ||
      (u0 % 4) != 0)
    return false;
  if (((uintptr_t)W % 16) != 0 || ((uintptr_t)mask % 4) != 0) return false;
  for (const float* p : {Zhi, Zlo, Rhi, Rlo})
    if (((uintptr_t)p % 16) != 0) return false;
  CUtensorMap maps[5];
  if (!encode_f32(&maps[0], Zhi, Bp, c, ldz, TK, TM) || !encode_f32(&maps[1], Zlo, Bp, c, ldz, TK, TM) ||
      !encode_f32(&maps[2], Rhi, Bp, b, ldz, TK, TN) || !encode_f32(&maps[3], Rlo, Bp, b, ldz, TK, TN) ||
      !encode_f32(&maps[4], W, b, c, ldw, 32, TM))
    return false;
  if (score == kWanda)
    *err = launch_variant<kWanda>(maps, c, b, u0, j, Bp, upper ? 1 : 0, mask, sc, hist_end, hist1, ctl, l2, pk, st, s,
                                  spare_sms, -1);
  else if (score == kObs)
    *err = launch_variant<kObs>(maps, c, b, u0, j, Bp, upper ? 1 : 0, mask, sc, hist_end, hist1, ctl, l2, pk, st, s,
                                spare_sms, -1);
  else
    *err = launch_variant<kNoScore>(maps, c, b, u0, j, Bp, upper ? 1 : 0, mask, sc, hist_end, hist1, ctl, l2, pk, st, s,
                                    spare_sms, keep);
  return true;
}

}  // namespace pwp
