// bat_attention_forward_noalloc: the forward for callers that cannot allocate device memory.
//
// Who needs it: a process whose device memory is entirely owned by another allocator (for
// example a framework caching allocator that reserved the pool up front, so a cudaMalloc from
// this library would fail or fragment it), or a latency-critical serving loop that must not
// call cudaMalloc/cudaFree because they can synchronize the whole device.  Such callers can
// still create their plans once at set-up time; per call they only pass inputs and outputs.
//
// What it does: runs exactly bat_attention_forward, with the split-path scratch (per-chunk
// partial outputs and log-sum-exps) placed in a fixed array compiled into the library instead
// of a caller-supplied workspace.  Nothing is allocated by the call.
//
// Limits and sharing:
//   * the array holds kNoAllocScratchBytes (32 MiB); a plan that needs more scratch is
//     rejected with BAT_ERR_INVALID_ARG and a message naming both sizes;
//   * every GPU that loads the library keeps this array until the process exits;
//   * all calls on a device share the one array: calls whose kernels overlap on the GPU (on
//     different streams, for example) race on it.  Serialize them on one stream;
//   * the array keeps whatever the last call left.  Nothing needs to start at zero: every
//     partial slot a split plan reads is written earlier in the same call;
//   * the first call on each device resolves the array's device address (with that device
//     current); make that first call before any stream capture begins on the device.  The
//     address is kept for the life of the process; cudaDeviceReset unloads the library's device
//     code, after which the kept address is stale, so this entry point must not be called again
//     on a device that was reset.
#include <cuda_runtime.h>

#include <cstdio>
#include <mutex>

#include "bat.h"

namespace {

constexpr size_t kNoAllocScratchBytes = 32u << 20;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {nullptr};

}  // namespace

namespace bat {
void set_last_error(const char* msg);
}

extern "C" bat_status bat_attention_forward_noalloc(const bat_plan* plan, const void* q, const void* k_suf,
                                                    const void* v_suf, const void* k_cache, const void* v_cache,
                                                    float scale, bat_dtype dt, void* out, float* lse, void* stream) {
  if (!plan) return bat_attention_forward(plan, q, k_suf, v_suf, k_cache, v_cache, scale, dt, out, lse, nullptr, 0,
                                          stream);
  const size_t need = bat_workspace_bytes(plan);
  if (need > kNoAllocScratchBytes) {
    char msg[256];
    snprintf(msg, sizeof(msg),
             "bat_attention_forward_noalloc: the plan needs %zu bytes of split scratch, more than the fixed %zu "
             "bytes; use bat_attention_forward with a caller-allocated workspace",
             need, kNoAllocScratchBytes);
    bat::set_last_error(msg);
    return BAT_ERR_INVALID_ARG;
  }
  void* scratch = nullptr;
  if (need > 0) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
      bat::set_last_error("bat_attention_forward_noalloc: no usable current device");
      return BAT_ERR_CUDA;
    }
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_ptr[dev]) {
      // Host code cannot use the array's name as a device address (in host code it names a
      // host-side stand-in): ask the runtime for it, once per device, with that device current.
      void* p = nullptr;
      e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
      if (e != cudaSuccess || !p) {
        char msg[256];
        snprintf(msg, sizeof(msg), "bat_attention_forward_noalloc: cudaGetSymbolAddress failed: %s",
                 cudaGetErrorString(e));
        bat::set_last_error(msg);
        return BAT_ERR_CUDA;
      }
      g_scratch_ptr[dev] = p;
    }
    scratch = g_scratch_ptr[dev];
  }
  return bat_attention_forward(plan, q, k_suf, v_suf, k_cache, v_cache, scale, dt, out, lse, scratch,
                               need > 0 ? kNoAllocScratchBytes : 0, stream);
}
