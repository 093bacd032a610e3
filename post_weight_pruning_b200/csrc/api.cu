// C ABI of libpwp: argument checks, workspace layout and the launch sequence.
// The declarations and their contracts are in include/pwp.h.
#include <cstring>

#include "pwp_internal.cuh"

namespace pwp {
struct PruneBuffers;
size_t prune_ws_layout(const pwp_config* cfg, int c, int b, PruneBuffers* pb, char* base);
cudaError_t launch_prune(const pwp_config* cfg, const void* W, int wtype, int c, int b, float* H,
                         float* Wout, uint8_t* mask, void* ws, pwp_stats* st, cudaStream_t s,
                         bool stats_ready);
cudaError_t launch_hessian_simt(const void* X, int xtype, long long n, int b, float* H, int beta,
                                cudaStream_t s);
cudaError_t launch_hessian_tc(const void* X, long long n, int b, float* H, int beta, cudaStream_t s,
                              bool* used, pwp_stats* st);
cudaError_t launch_stats_init(pwp_stats* st, cudaStream_t s);
cudaError_t sweep_step(const pwp_config* cfg, const void* W, int wtype, int c, int b, long long c_budget, float* H,
                       float* Wout, uint8_t* mask, void* ws, pwp_stats* st, const unsigned int* ties_all, int world,
                       int rank, cudaStream_t s, int step, int t);
void sweep_buffers(const pwp_config* cfg, int c, int b, void* ws, unsigned int** level1, long long* n1,
                   unsigned int** level2, long long* n2, unsigned int** ties, long long* nt);
}  // namespace pwp

using namespace pwp;

static bool valid_dtype(int32_t t) { return t == PWP_BF16 || t == PWP_FP32; }

static bool valid_cfg(const pwp_config* cfg, int32_t c, int32_t b) {
  if (!cfg) return false;
  if (c < 1 || b < 1 || b > 16384) return false;
  if ((long long)c * (long long)b >= (1LL << 31)) return false;
  if (cfg->method < PWP_THANOS || cfg->method > PWP_MAGNITUDE) return false;
  const bool second_order = cfg->method == PWP_THANOS || cfg->method == PWP_SPARSEGPT;
  if (second_order && (cfg->block < 1 || cfg->block > kMaxBlock)) return false;
  if (second_order && !(cfg->damp >= 0.f && cfg->damp < 1e30f)) return false;
  if (!(cfg->alpha >= 0.f && cfg->alpha < 1.f) || (!second_order && cfg->alpha != 0.f)) return false;
  if (cfg->pattern == PWP_UNSTRUCTURED) {
    if (!(cfg->sparsity >= 0.f && cfg->sparsity < 1.f)) return false;
  } else if (cfg->pattern == PWP_NM) {
    const int n = cfg->nm_n, m = cfg->nm_m;
    if (m < 2 || m > 32 || (m & (m - 1)) != 0) return false;  // m must divide a warp
    if (n < 1 || n >= m) return false;
    if (b % m != 0 || (second_order && cfg->block % m != 0)) return false;
  } else {
    return false;
  }
  return true;
}

static bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

extern "C" {

const char* pwp_status_string(int32_t status) {
  switch (status) {
    case PWP_OK: return "ok";
    case PWP_EINVAL: return "invalid argument";
    case PWP_ENOTSPD: return "damped Hessian is not positive definite";
    case PWP_EWORKSPACE: return "workspace missing, misaligned or too small";
    case PWP_ECUDA: return "CUDA error";
    case PWP_ETIMEOUT: return "bounded device-side wait timed out";
    case PWP_EBUDGET: return "sparsity target could not be met";
    default: return "unknown status";
  }
}

int32_t pwp_version(void) { return 200; }

size_t pwp_workspace_bytes(const pwp_config* cfg, int32_t c, int32_t b) {
  if (!valid_cfg(cfg, c, b)) return 0;
  return prune_ws_layout(cfg, c, b, nullptr, nullptr);
}

size_t pwp_factor_workspace_bytes(int32_t b) {
  if (b < 1 || b > 16384) return 0;
  return factor_ws_bytes(b);
}

// H := beta*H + 2 X X^T; device-side failures go to st when it is given.
static pwp_status hessian_impl(const void* X, int32_t xtype, int64_t n, int32_t b, float* H, int32_t beta,
                               pwp_stats* st, cudaStream_t s) {
  cudaError_t e = cudaSuccess;
  bool used = false;
  prof_begin(kKHessian, s);
  if (xtype == PWP_BF16) {
    e = launch_hessian_tc(X, n, b, H, beta, s, &used, st);
    if (e != cudaSuccess) return PWP_ECUDA;
  }
  if (!used) e = launch_hessian_simt(X, xtype, n, b, H, beta, s);
  prof_end(kKHessian, s);
  count_launches(1);
  return e == cudaSuccess ? PWP_OK : PWP_ECUDA;
}

pwp_status pwp_hessian_accumulate(const void* X, int32_t xtype, int64_t n, int32_t b, float* H,
                                  int32_t beta, void* stream) {
  if (!H || b < 1 || b > 16384 || n < 0 || (n > 0 && !X) || !valid_dtype(xtype) ||
      (beta != 0 && beta != 1))
    return PWP_EINVAL;
  return hessian_impl(X, xtype, n, b, H, beta, nullptr, (cudaStream_t)stream);
}

pwp_status pwp_damp_factor(float* H, int32_t b, float damp, float* g_diag, void* ws, size_t ws_bytes,
                           pwp_stats* st, void* stream) {
  if (!H || !g_diag || !st || b < 1 || b > 16384 || !(damp >= 0.f)) return PWP_EINVAL;
  if (!ws || !aligned(ws, 256) || ws_bytes < factor_ws_bytes(b)) return PWP_EWORKSPACE;
  cudaStream_t s = (cudaStream_t)stream;
  if (cudaMemsetAsync(st, 0, sizeof(pwp_stats), s) != cudaSuccess) return PWP_ECUDA;
  cudaError_t e = launch_damp_factor(H, b, damp, g_diag, ws, ws_bytes, st, s);
  return e == cudaSuccess ? PWP_OK : PWP_ECUDA;
}

pwp_status pwp_prune_layer(const pwp_config* cfg, const void* W, int32_t wtype, int32_t c, int32_t b,
                           float* H, float* W_out, uint8_t* mask, void* ws, size_t ws_bytes,
                           pwp_stats* st, void* stream) {
  if (!valid_cfg(cfg, c, b) || !valid_dtype(wtype) || !W || !W_out || !mask || !st) return PWP_EINVAL;
  if (!H && cfg->method != PWP_MAGNITUDE) return PWP_EINVAL;
  if (!ws || !aligned(ws, 256) || ws_bytes < prune_ws_layout(cfg, c, b, nullptr, nullptr))
    return PWP_EWORKSPACE;
  cudaError_t e = launch_prune(cfg, W, wtype, c, b, H, W_out, mask, ws, st, (cudaStream_t)stream, false);
  return e == cudaSuccess ? PWP_OK : PWP_ECUDA;
}

pwp_status pwp_prune_layer_x(const pwp_config* cfg, const void* W, int32_t wtype, int32_t c, int32_t b,
                             const void* X, int32_t xtype, int64_t n, float* H, float* W_out,
                             uint8_t* mask, void* ws, size_t ws_bytes, pwp_stats* st, void* stream) {
  const bool no_update = valid_cfg(cfg, c, b) && (cfg->method == PWP_WANDA || cfg->method == PWP_MAGNITUDE);
  if (!valid_cfg(cfg, c, b) || !valid_dtype(wtype) || !valid_dtype(xtype) || !W || (!H && !no_update) ||
      !W_out || !mask || !st || n < 0 || (n > 0 && !X))
    return PWP_EINVAL;
  if (!ws || !aligned(ws, 256) || ws_bytes < prune_ws_layout(cfg, c, b, nullptr, nullptr))
    return PWP_EWORKSPACE;
  cudaStream_t s = (cudaStream_t)stream;
  if (no_update) {
    cudaError_t e = launch_no_update(cfg, W, wtype, c, b, nullptr, X, xtype, n, W_out, mask, ws, st, false, s);
    return e == cudaSuccess ? PWP_OK : PWP_ECUDA;
  }
  if (launch_stats_init(st, s) != cudaSuccess) return PWP_ECUDA;
  pwp_status ps = hessian_impl(X, xtype, n, b, H, 0, st, s);
  if (ps != PWP_OK) return ps;
  cudaError_t e = launch_prune(cfg, W, wtype, c, b, H, W_out, mask, ws, st, s, true);
  return e == cudaSuccess ? PWP_OK : PWP_ECUDA;
}

static size_t dtype_bytes(int32_t t) { return t == PWP_BF16 ? 2 : 4; }

pwp_status pwp_prune_layer_host(const pwp_config* cfg, const void* W_host, int32_t wtype, int32_t c, int32_t b,
                                const void* X_host, int32_t xtype, int64_t n, void* W_dev, void* X_dev,
                                float* H_dev, float* W_out_dev, uint8_t* mask_dev, float* W_out_host,
                                uint8_t* mask_out_host, void* ws, size_t ws_bytes, pwp_stats* st, void* stream) {
  const bool no_update = valid_cfg(cfg, c, b) && (cfg->method == PWP_WANDA || cfg->method == PWP_MAGNITUDE);
  if (!valid_cfg(cfg, c, b) || !valid_dtype(wtype) || !valid_dtype(xtype) || !W_host || !W_dev ||
      (!H_dev && !no_update) || !W_out_dev || !mask_dev || !W_out_host || !mask_out_host || !st || n < 0 ||
      (n > 0 && (!X_host || !X_dev)))
    return PWP_EINVAL;
  if (!ws || !aligned(ws, 256) || ws_bytes < prune_ws_layout(cfg, c, b, nullptr, nullptr))
    return PWP_EWORKSPACE;
  cudaStream_t s = (cudaStream_t)stream;
  // a copy stream and two events of this call's own (released once their work is done)
  cudaStream_t cp = nullptr;
  cudaEvent_t ev = nullptr, ev_w = nullptr;
  if (cudaStreamCreateWithFlags(&cp, cudaStreamNonBlocking) != cudaSuccess) return PWP_ECUDA;
  cudaError_t e = cudaEventCreateWithFlags(&ev, cudaEventDisableTiming);
  if (e == cudaSuccess) e = cudaEventCreateWithFlags(&ev_w, cudaEventDisableTiming);
  // the copies start after the caller's earlier work on `stream`
  if (e == cudaSuccess) e = cudaEventRecord(ev, s);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(cp, ev, 0);
  if (e == cudaSuccess) e = launch_stats_init(st, s);
  pwp_status ps = e == cudaSuccess ? PWP_OK : PWP_ECUDA;
  const size_t xrow = (size_t)b * dtype_bytes(xtype);
  if (ps == PWP_OK && no_update) {
    // Wanda and magnitude: no Hessian; X (Wanda's column norms) and W, then the prune
    if (n > 0) e = cudaMemcpyAsync(X_dev, X_host, (size_t)n * xrow, cudaMemcpyHostToDevice, cp);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(W_dev, W_host, (size_t)c * b * dtype_bytes(wtype), cudaMemcpyHostToDevice, cp);
    if (e == cudaSuccess) e = cudaEventRecord(ev, cp);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(s, ev, 0);
    if (e == cudaSuccess)
      e = launch_no_update(cfg, W_dev, wtype, c, b, nullptr, cfg->method == PWP_WANDA ? X_dev : nullptr, xtype,
                           cfg->method == PWP_WANDA ? n : 0, W_out_dev, mask_dev, ws, st, true, s);
    if (e != cudaSuccess) ps = PWP_ECUDA;
  } else if (ps == PWP_OK) {
    // X in row chunks, each folded into H as soon as it lands; then W, which the prune first
    // needs after the factor
    const int64_t nch = n >= 8 * 1024 ? 8 : 1;
    const int64_t rows = (n + nch - 1) / nch;
    for (int64_t r0 = 0; r0 < n && ps == PWP_OK; r0 += rows) {
      const int64_t nr = n - r0 < rows ? n - r0 : rows;
      e = cudaMemcpyAsync((char*)X_dev + (size_t)r0 * xrow, (const char*)X_host + (size_t)r0 * xrow,
                          (size_t)nr * xrow, cudaMemcpyHostToDevice, cp);
      if (e == cudaSuccess) e = cudaEventRecord(ev, cp);
      if (e == cudaSuccess) e = cudaStreamWaitEvent(s, ev, 0);
      if (e != cudaSuccess) {
        ps = PWP_ECUDA;
        break;
      }
      ps = hessian_impl((const char*)X_dev + (size_t)r0 * xrow, xtype, nr, b, H_dev, r0 > 0 ? 1 : 0, st, s);
    }
    if (ps == PWP_OK && n == 0) e = cudaMemsetAsync(H_dev, 0, (size_t)b * b * sizeof(float), s);
    if (ps == PWP_OK && e == cudaSuccess)
      e = cudaMemcpyAsync(W_dev, W_host, (size_t)c * b * dtype_bytes(wtype), cudaMemcpyHostToDevice, cp);
    if (ps == PWP_OK && e == cudaSuccess) e = cudaEventRecord(ev_w, cp);
    if (ps == PWP_OK && e == cudaSuccess) e = cudaStreamWaitEvent(s, ev_w, 0);
    // finished column blocks go back during the sweep (not for outlier rows, whose compact
    // prune is scattered back at the end)
    const HostOut ho{W_out_host, mask_out_host, cp, ev};
    const bool blockwise = cfg->alpha == 0.f;
    if (ps == PWP_OK && e == cudaSuccess)
      e = launch_prune_out(cfg, W_dev, wtype, c, b, H_dev, W_out_dev, mask_dev, ws, st, s, true,
                           blockwise ? &ho : nullptr);
    if (e != cudaSuccess) ps = PWP_ECUDA;
    if (ps == PWP_OK && blockwise) {
      // the outputs are on their way; `stream` waits for the last copies
      e = cudaEventRecord(ev, cp);
      if (e == cudaSuccess) e = cudaStreamWaitEvent(s, ev, 0);
      if (e != cudaSuccess) ps = PWP_ECUDA;
      cudaEventDestroy(ev);
      cudaEventDestroy(ev_w);
      cudaStreamDestroy(cp);
      return ps;
    }
  }
  if (ps == PWP_OK) {
    e = cudaMemcpyAsync(W_out_host, W_out_dev, (size_t)c * b * sizeof(float), cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaMemcpyAsync(mask_out_host, mask_dev, (size_t)c * b, cudaMemcpyDeviceToHost, s);
    if (e != cudaSuccess) ps = PWP_ECUDA;
  }
  // `stream` waits for whatever the copy stream still has, on the error paths too
  if (ev && cudaEventRecord(ev, cp) == cudaSuccess) cudaStreamWaitEvent(s, ev, 0);
  if (ev) cudaEventDestroy(ev);
  if (ev_w) cudaEventDestroy(ev_w);
  cudaStreamDestroy(cp);
  return ps;
}

// Device memory of pwp_prune_layers_host, in order (each piece 256-byte aligned): two W
// buffers, two X buffers, H, two W-hat buffers, two masks, the prune workspace.
static size_t layers_host_layout(const pwp_config* cfg, int32_t c, int32_t b, int64_t n, int32_t wtype,
                                 int32_t xtype, size_t* off) {
  auto up = [](size_t v) { return (v + 255) & ~(size_t)255; };
  const size_t wb = up((size_t)c * b * dtype_bytes(wtype)), xb = up((size_t)n * b * dtype_bytes(xtype));
  const size_t hb = up((size_t)b * b * sizeof(float)), ob = up((size_t)c * b * sizeof(float)), mb = up((size_t)c * b);
  const size_t sizes[10] = {wb, wb, xb, xb, hb, ob, ob, mb, mb, prune_ws_layout(cfg, c, b, nullptr, nullptr)};
  size_t at = 0;
  for (int i = 0; i < 10; ++i) {
    if (off) off[i] = at;
    at += up(sizes[i]);
  }
  return at;
}

size_t pwp_layers_host_bytes(const pwp_config* cfg, int32_t c, int32_t b, int64_t n, int32_t wtype, int32_t xtype) {
  if (!valid_cfg(cfg, c, b) || !valid_dtype(wtype) || !valid_dtype(xtype) || n < 0) return 0;
  return layers_host_layout(cfg, c, b, n, wtype, xtype, nullptr);
}

pwp_status pwp_prune_layers_host(const pwp_config* cfg, int32_t nlayers, const void* const* W_host, int32_t wtype,
                                 int32_t c, int32_t b, const void* const* X_host, int32_t xtype, int64_t n,
                                 float* const* W_out_host, uint8_t* const* mask_out_host, void* dev,
                                 size_t dev_bytes, pwp_stats* st, void* stream) {
  if (!valid_cfg(cfg, c, b) || !valid_dtype(wtype) || !valid_dtype(xtype) || nlayers < 0 || n < 0 || !W_host ||
      !W_out_host || !mask_out_host || !st || (n > 0 && !X_host))
    return PWP_EINVAL;
  for (int i = 0; i < nlayers; ++i)
    if (!W_host[i] || !W_out_host[i] || !mask_out_host[i] || (n > 0 && !X_host[i])) return PWP_EINVAL;
  size_t off[10];
  if (!dev || !aligned(dev, 256) || dev_bytes < layers_host_layout(cfg, c, b, n, wtype, xtype, off))
    return PWP_EWORKSPACE;
  if (nlayers == 0) return PWP_OK;
  const bool no_update = cfg->method == PWP_WANDA || cfg->method == PWP_MAGNITUDE;
  char* base = (char*)dev;
  void* W_dev[2] = {base + off[0], base + off[1]};
  void* X_dev[2] = {base + off[2], base + off[3]};
  float* H_dev = (float*)(base + off[4]);
  float* Wo_dev[2] = {(float*)(base + off[5]), (float*)(base + off[6])};
  uint8_t* mk_dev[2] = {(uint8_t*)(base + off[7]), (uint8_t*)(base + off[8])};
  void* ws = base + off[9];
  cudaStream_t s = (cudaStream_t)stream;
  // an input and an output copy stream and the events of this call (released once their
  // work is done): a layer's inputs go in while the previous layer is pruned, its results
  // come back while the next one is
  constexpr int kChunks = 8;
  cudaStream_t cin = nullptr, cout = nullptr;
  cudaEvent_t ev_start = nullptr, ev_chunk[kChunks] = {}, ev_w = nullptr, ev_blk = nullptr, ev_in_free[2] = {},
              ev_out_done[2] = {};
  cudaError_t e = cudaStreamCreateWithFlags(&cin, cudaStreamNonBlocking);
  if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&cout, cudaStreamNonBlocking);
  for (cudaEvent_t* ev : {&ev_start, &ev_w, &ev_blk, &ev_in_free[0], &ev_in_free[1], &ev_out_done[0],
                          &ev_out_done[1]})
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(ev, cudaEventDisableTiming);
  for (int i = 0; i < kChunks && e == cudaSuccess; ++i) e = cudaEventCreateWithFlags(&ev_chunk[i], cudaEventDisableTiming);
  // the copies start after the caller's earlier work on `stream`
  if (e == cudaSuccess) e = cudaEventRecord(ev_start, s);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(cin, ev_start, 0);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(cout, ev_start, 0);
  pwp_status ps = e == cudaSuccess ? PWP_OK : PWP_ECUDA;
  const size_t xrow = (size_t)b * dtype_bytes(xtype), wbytes = (size_t)c * b * dtype_bytes(wtype);
  const int64_t nch = (!no_update && n >= 8 * 1024) ? kChunks : 1;
  const int64_t rows = n > 0 ? (n + nch - 1) / nch : 0;
  for (int i = 0; i < nlayers && ps == PWP_OK; ++i) {
    const int k = i & 1;
    pwp_stats* sti = st + i;
    // inputs of layer i into set k, once layer i-2 is done with it
    if (i >= 2) e = cudaStreamWaitEvent(cin, ev_in_free[k], 0);
    int nchunks = 0;
    for (int64_t r0 = 0; r0 < n && e == cudaSuccess; r0 += rows, ++nchunks) {
      const int64_t nr = n - r0 < rows ? n - r0 : rows;
      e = cudaMemcpyAsync((char*)X_dev[k] + (size_t)r0 * xrow, (const char*)X_host[i] + (size_t)r0 * xrow,
                          (size_t)nr * xrow, cudaMemcpyHostToDevice, cin);
      if (e == cudaSuccess) e = cudaEventRecord(ev_chunk[nchunks], cin);
    }
    if (e == cudaSuccess) e = cudaMemcpyAsync(W_dev[k], W_host[i], wbytes, cudaMemcpyHostToDevice, cin);
    if (e == cudaSuccess) e = cudaEventRecord(ev_w, cin);
    if (e == cudaSuccess) e = launch_stats_init(sti, s);
    // W-hat and the mask of set k are free once layer i-2's results are back
    if (e == cudaSuccess && i >= 2) e = cudaStreamWaitEvent(s, ev_out_done[k], 0);
    if (e != cudaSuccess) {
      ps = PWP_ECUDA;
      break;
    }
    if (no_update) {
      for (int ch = 0; ch < nchunks && e == cudaSuccess; ++ch) e = cudaStreamWaitEvent(s, ev_chunk[ch], 0);
      if (e == cudaSuccess) e = cudaStreamWaitEvent(s, ev_w, 0);
      if (e == cudaSuccess)
        e = launch_no_update(cfg, W_dev[k], wtype, c, b, nullptr, cfg->method == PWP_WANDA ? X_dev[k] : nullptr,
                             xtype, cfg->method == PWP_WANDA ? n : 0, Wo_dev[k], mk_dev[k], ws, sti, true, s);
      if (e == cudaSuccess) e = cudaEventRecord(ev_in_free[k], s);
    } else {
      // each chunk of X folded into H as soon as it lands
      int ch = 0;
      for (int64_t r0 = 0; r0 < n && ps == PWP_OK; r0 += rows, ++ch) {
        const int64_t nr = n - r0 < rows ? n - r0 : rows;
        e = cudaStreamWaitEvent(s, ev_chunk[ch], 0);
        if (e != cudaSuccess) {
          ps = PWP_ECUDA;
          break;
        }
        ps = hessian_impl((const char*)X_dev[k] + (size_t)r0 * xrow, xtype, nr, b, H_dev, r0 > 0 ? 1 : 0, sti, s);
      }
      if (ps != PWP_OK) break;
      if (n == 0) e = cudaMemsetAsync(H_dev, 0, (size_t)b * b * sizeof(float), s);
      if (e == cudaSuccess) e = cudaStreamWaitEvent(s, ev_w, 0);
      const HostOut ho{W_out_host[i], mask_out_host[i], cout, ev_blk};
      const bool blockwise = cfg->alpha == 0.f;
      if (e == cudaSuccess)
        e = launch_prune_out(cfg, W_dev[k], wtype, c, b, H_dev, Wo_dev[k], mk_dev[k], ws, sti, s, true,
                             blockwise ? &ho : nullptr);
      if (e == cudaSuccess) e = cudaEventRecord(ev_in_free[k], s);
      if (e == cudaSuccess && !blockwise) {
        // outlier rows: the whole result once the prune is done
        e = cudaStreamWaitEvent(cout, ev_in_free[k], 0);
        if (e == cudaSuccess)
          e = cudaMemcpyAsync(W_out_host[i], Wo_dev[k], (size_t)c * b * sizeof(float), cudaMemcpyDeviceToHost, cout);
        if (e == cudaSuccess)
          e = cudaMemcpyAsync(mask_out_host[i], mk_dev[k], (size_t)c * b, cudaMemcpyDeviceToHost, cout);
      }
    }
    if (e == cudaSuccess && no_update) {
      e = cudaStreamWaitEvent(cout, ev_in_free[k], 0);
      if (e == cudaSuccess)
        e = cudaMemcpyAsync(W_out_host[i], Wo_dev[k], (size_t)c * b * sizeof(float), cudaMemcpyDeviceToHost, cout);
      if (e == cudaSuccess) e = cudaMemcpyAsync(mask_out_host[i], mk_dev[k], (size_t)c * b, cudaMemcpyDeviceToHost, cout);
    }
    if (e == cudaSuccess) e = cudaEventRecord(ev_out_done[k], cout);
    if (e != cudaSuccess) ps = PWP_ECUDA;
  }
  // `stream` waits for the last copies either way
  if (cudaEventRecord(ev_start, cout) == cudaSuccess) cudaStreamWaitEvent(s, ev_start, 0);
  if (cudaEventRecord(ev_w, cin) == cudaSuccess) cudaStreamWaitEvent(s, ev_w, 0);
  for (cudaEvent_t ev : {ev_start, ev_w, ev_blk, ev_in_free[0], ev_in_free[1], ev_out_done[0], ev_out_done[1]})
    if (ev) cudaEventDestroy(ev);
  for (cudaEvent_t ev : ev_chunk)
    if (ev) cudaEventDestroy(ev);
  if (cin) cudaStreamDestroy(cin);
  if (cout) cudaStreamDestroy(cout);
  return ps;
}

pwp_status pwp_pack_24(const float* W_hat, const uint8_t* mask, int32_t c, int32_t b, uint16_t* values,
                       uint32_t* meta, pwp_stats* st, void* stream) {
  if (!W_hat || !mask || !values || !meta || !st || c < 1 || b < 4 || b > 16384 || (b % 4) != 0 ||
      (long long)c * (long long)b >= (1LL << 31) || !aligned(W_hat, 16) || !aligned(mask, 4))
    return PWP_EINVAL;
  cudaStream_t s = (cudaStream_t)stream;
  if (cudaMemsetAsync(st, 0, sizeof(pwp_stats), s) != cudaSuccess) return PWP_ECUDA;
  cudaError_t e = launch_pack24(W_hat, mask, c, b, values, meta, st, s);
  return e == cudaSuccess ? PWP_OK : PWP_ECUDA;
}

// The stepwise sweep: argument checks shared by both calls.
static pwp_status sweep_check(const pwp_sweep* a) {
  if (!a || !valid_cfg(a->cfg, a->c, a->b) || !valid_dtype(a->wtype)) return PWP_EINVAL;
  const pwp_config* cfg = a->cfg;
  if ((cfg->method != PWP_THANOS && cfg->method != PWP_SPARSEGPT) || cfg->pattern != PWP_UNSTRUCTURED ||
      cfg->alpha != 0.f)
    return PWP_EINVAL;
  if (a->c_total < a->c || a->c_total * (long long)a->b >= (1LL << 31) || a->world < 1 || a->rank < 0 ||
      a->rank >= a->world)
    return PWP_EINVAL;
  if (!a->ws || !aligned(a->ws, 256) || a->ws_bytes < prune_ws_layout(cfg, a->c, a->b, nullptr, nullptr))
    return PWP_EWORKSPACE;
  return PWP_OK;
}

pwp_status pwp_sweep_step(const pwp_sweep* a, int32_t step, int32_t t) {
  pwp_status ps = sweep_check(a);
  if (ps != PWP_OK) return ps;
  if (!a->W_dev || !a->H_dev || !a->W_out_dev || !a->mask_dev || !a->stats_dev) return PWP_EINVAL;
  const int nblk = (a->b + a->cfg->block - 1) / a->cfg->block;
  if (step < PWP_SWEEP_SETUP || step > PWP_SWEEP_FINISH) return PWP_EINVAL;
  if (step != PWP_SWEEP_SETUP && step != PWP_SWEEP_FINISH && (t < 0 || t >= nblk)) return PWP_EINVAL;
  if (step == PWP_SWEEP_CUT_TIES && !a->ties_all_dev) return PWP_EINVAL;
  cudaError_t e = sweep_step(a->cfg, a->W_dev, a->wtype, a->c, a->b, a->c_total, a->H_dev, a->W_out_dev, a->mask_dev,
                             a->ws, a->stats_dev, a->ties_all_dev, a->world, a->rank, (cudaStream_t)a->stream, step, t);
  return e == cudaSuccess ? PWP_OK : PWP_ECUDA;
}

pwp_status pwp_sweep_buffers(const pwp_sweep* a, uint32_t** level1, int64_t* n_level1, uint32_t** level2,
                             int64_t* n_level2, uint32_t** ties, int64_t* n_ties) {
  pwp_status ps = sweep_check(a);
  if (ps != PWP_OK) return ps;
  if (!level1 || !n_level1 || !level2 || !n_level2 || !ties || !n_ties) return PWP_EINVAL;
  long long n1, n2, nt;
  unsigned int *p1, *p2, *pt;
  sweep_buffers(a->cfg, a->c, a->b, a->ws, &p1, &n1, &p2, &n2, &pt, &nt);
  *level1 = p1;
  *n_level1 = n1;
  *level2 = p2;
  *n_level2 = n2;
  *ties = pt;
  *n_ties = nt;
  return PWP_OK;
}

}  // extern "C"
