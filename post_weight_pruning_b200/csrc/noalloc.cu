// pwp_prune_layer_noalloc: the layer prune for callers that cannot provide a workspace.
//
// Who needs this: some host programs cannot allocate device memory for this library
// at the time they call it -- for instance an operator plugged into an inference or
// training runtime that only hands the operator its input and output buffers, or a
// process whose device memory is fully owned by a framework's caching allocator, where
// an outside cudaMalloc either fails or is forbidden once the job is running.  Those
// callers still own W, H, W_out, mask and stats, but have no way to pass scratch.
//
// This entry point takes its scratch from one file-scope device array instead.  The
// array is part of the loaded module, so every GPU on which the library is used holds
// PWP_NOALLOC_SCRATCH_BYTES of it until the process exits.  No call here allocates or
// frees memory; the kernels are the same ones pwp_prune_layer launches.
#include <cuda.h>

#include <mutex>

#include "pwp_internal.cuh"

namespace pwp {
struct PruneBuffers;
size_t prune_ws_layout(const pwp_config* cfg, int c, int b, PruneBuffers* pb, char* base);
cudaError_t launch_prune(const pwp_config* cfg, const void* W, int wtype, int c, int b, float* H,
                         float* Wout, uint8_t* mask, void* ws, pwp_stats* st, cudaStream_t s,
                         bool stats_ready);
}  // namespace pwp

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[PWP_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};
unsigned long long g_scratch_ctx[kMaxDevices] = {};   // id of the context the address belongs to

// Unique id of the calling thread's current context (0 if there is none yet, or if the
// driver does not provide the calls).  Ids are never reused within a process, so a
// context created after cudaDeviceReset differs.  The two driver calls are reached through
// the runtime's entry-point lookup, so the library does not link the driver library.
unsigned long long current_context_id() {
  using GetCurrent = CUresult (*)(CUcontext*);
  using GetId = CUresult (*)(CUcontext, unsigned long long*);
  static const GetCurrent get_current = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    return (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess) ? reinterpret_cast<GetCurrent>(p) : (GetCurrent) nullptr;
  }();
  static const GetId get_id = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    return (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess) ? reinterpret_cast<GetId>(p) : (GetId) nullptr;
  }();
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx) return 0;
  if (get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

// The host-side name g_noalloc_scratch is only a stand-in for the symbol, not a device
// address: the device address is looked up with the device current, once per device and
// context (again after a device reset, whose new context reloads the module).
cudaError_t scratch_for_current_device(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  const unsigned long long id = current_context_id();
  if (!g_scratch_addr[dev] || id == 0 || id != g_scratch_ctx[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);   // also creates the context if needed
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = p;
    g_scratch_ctx[dev] = current_context_id();
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" pwp_status pwp_prune_layer_noalloc(const pwp_config* cfg, const void* W, int32_t wtype,
                                              int32_t c, int32_t b, float* H, float* W_out,
                                              uint8_t* mask, pwp_stats* st, void* stream) {
  // same argument contract as pwp_prune_layer
  size_t need = pwp_workspace_bytes(cfg, c, b);
  if (need == 0 || (wtype != PWP_BF16 && wtype != PWP_FP32) || !W || (!H && cfg->method != PWP_MAGNITUDE) ||
      !W_out || !mask || !st)
    return PWP_EINVAL;
  if (need > (size_t)PWP_NOALLOC_SCRATCH_BYTES) return PWP_EWORKSPACE;
  void* ws = nullptr;
  if (scratch_for_current_device(&ws) != cudaSuccess) return PWP_ECUDA;
  cudaStream_t s = (cudaStream_t)stream;
  // The array keeps whatever the previous call left in it; start from zeros.
  if (cudaMemsetAsync(ws, 0, need, s) != cudaSuccess) return PWP_ECUDA;
  cudaError_t e = pwp::launch_prune(cfg, W, wtype, c, b, H, W_out, mask, ws, st, s, false);
  return e == cudaSuccess ? PWP_OK : PWP_ECUDA;
}
