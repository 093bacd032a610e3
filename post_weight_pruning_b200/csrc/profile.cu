// Launch counting and optional per-kernel-class CUDA-event timing.
#include <atomic>
#include <cstdio>
#include <cstdlib>
#include <vector>

#include "pwp_internal.cuh"

namespace pwp {

std::atomic<long long> g_launches{0};
constexpr long long kDefaultWaitLimit = 1ll << 26;
std::atomic<long long> g_wait_limit{kDefaultWaitLimit};

void count_launches(long long n) { g_launches += n; }

bool trace_launches() {
  static const bool on = [] {
    const char* v = std::getenv("PWP_TRACE");
    return v != nullptr && v[0] != '\0' && v[0] != '0';
  }();
  return on;
}

void trace_launch(const void* kernel, dim3 grid, dim3 block, size_t smem, cudaStream_t s, cudaError_t launched) {
  const char* name = nullptr;
  if (cudaFuncGetName(&name, kernel) != cudaSuccess || name == nullptr) name = "?";
  std::fprintf(stderr, "pwp launch %s grid (%u,%u,%u) block %u smem %zu: %s\n", name, grid.x, grid.y, grid.z,
               block.x, smem, cudaGetErrorString(launched));
  std::fflush(stderr);
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  cudaStreamIsCapturing(s, &cap);
  if (launched != cudaSuccess || cap != cudaStreamCaptureStatusNone) return;
  const cudaError_t e = cudaStreamSynchronize(s);
  std::fprintf(stderr, "pwp   done %s: %s\n", name, cudaGetErrorString(e));
  std::fflush(stderr);
}
long long wait_limit() { return g_wait_limit.load(); }

namespace {
struct Prof {
  int which = -1;
  int n = 0;
  std::vector<cudaEvent_t> ev0, ev1;
};
Prof g_prof;
}  // namespace

void prof_begin(int which, cudaStream_t s) {
  if (g_prof.which == which && g_prof.n < (int)g_prof.ev0.size()) cudaEventRecord(g_prof.ev0[g_prof.n], s);
}

void prof_end(int which, cudaStream_t s) {
  if (g_prof.which == which && g_prof.n < (int)g_prof.ev0.size()) {
    cudaEventRecord(g_prof.ev1[g_prof.n], s);
    ++g_prof.n;
  }
}

}  // namespace pwp

using namespace pwp;

extern "C" {

int64_t pwp_kernel_launches(void) { return g_launches.load(); }

int64_t pwp_set_wait_limit(int64_t polls) {
  return g_wait_limit.exchange(polls < 0 ? kDefaultWaitLimit : (long long)polls);
}

int32_t pwp_profile_enable(int32_t which, int32_t capacity) {
  for (auto e : g_prof.ev0) cudaEventDestroy(e);
  for (auto e : g_prof.ev1) cudaEventDestroy(e);
  g_prof.ev0.clear();
  g_prof.ev1.clear();
  g_prof.n = 0;
  g_prof.which = -1;
  if (which < 0 || capacity <= 0) return PWP_OK;
  g_prof.ev0.resize(capacity);
  g_prof.ev1.resize(capacity);
  for (int i = 0; i < capacity; ++i) {
    if (cudaEventCreate(&g_prof.ev0[i]) != cudaSuccess || cudaEventCreate(&g_prof.ev1[i]) != cudaSuccess)
      return PWP_ECUDA;
  }
  g_prof.which = which;
  return PWP_OK;
}

int32_t pwp_profile_read(float* ms, int32_t cap) {
  int n = g_prof.n < cap ? g_prof.n : cap;
  for (int i = 0; i < n; ++i) {
    if (cudaEventSynchronize(g_prof.ev1[i]) != cudaSuccess) return -1;
    float t = 0.f;
    cudaEventElapsedTime(&t, g_prof.ev0[i], g_prof.ev1[i]);
    ms[i] = t;
  }
  g_prof.n = 0;
  return n;
}

}  // extern "C"
