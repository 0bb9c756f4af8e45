// Kernel parameter blocks and host-side launchers (internal to libbat.so).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include "bat_internal.h"

namespace bat {

// Device-side bounds checks of debug builds (-DBAT_DEBUG; the library is then libbat_debug.so).
// A failed check sets bit 1 of the device status word, records the check's code and the
// offending value in words 1 and 2 (the first failure wins), and the caller skips the access
// (stores) or clamps it into the tensor (loads, so every barrier still completes).  Nothing
// traps.  In normal builds a check is the constant `true` and costs nothing.
enum DebugCheck : uint32_t {
  kChkQLoad = 1,      // Q tile coordinates inside q
  kChkCacheLoad = 2,  // K/V tile coordinates inside the cache
  kChkSufLoad = 3,    // K/V tile coordinates inside k_suf / v_suf
  kChkOutBulk = 4,    // bulk store of 32 output rows inside out
  kChkOutRow = 5,     // one output row inside out
  kChkLse = 6,        // LSE element inside lse
  kChkPartial = 7,    // split partial row inside the workspace
  kChkItem = 8,       // work-item fields (head, query tiles, key ranges) inside the tensors
  kChkSimtRow = 9,    // fp32 path: a row it reads or writes
  kChkMerge = 10,     // merge: a partial it reads or a row it writes
};
#ifdef BAT_DEBUG
__device__ __forceinline__ bool debug_check(uint32_t* status, bool ok, uint32_t code, long long val) {
  if (!ok && status) {
    if (atomicCAS(status + 1, 0u, code) == 0u) atomicExch(status + 2, (uint32_t)val);
    atomicOr(status, 2u);
  }
  return ok;
}
#define BAT_DCHECK(status, cond, code, val) ::bat::debug_check((status), (cond), (code), (long long)(val))
#else
#define BAT_DCHECK(status, cond, code, val) true
#endif

// Tensor-core path (bf16 in, fp32 accumulate), d in {64, 128}.
struct alignas(64) TcParams {
  CUtensorMap tm_q, tm_ks, tm_vs, tm_kc, tm_vc;  // [T, H*d] 2-D maps, box 64 x 128, 128B swizzle
  CUtensorMap tm_o;     // output [T_suf, H*d], box 64 x 32 (one warp's rows), 128B swizzle
  const WorkItem* items;
  int64_t n_items;
  void* out;            // bf16 [T_suf, H, d]
  float* lse;           // fp32 [H, T_suf] or null
  float* part_o;        // fp32 [slots, 128, d] (split items)
  float* part_lse;      // fp32 [slots, 128], log2 units
  int32_t T_suf, H;
  float scale_log2;     // softmax scale * log2(e)
  int32_t pad0;
  uint32_t* status;     // device status words (bit 0 of word 0: a wait timed out; debug checks)
  uint64_t wait_ns;     // bound on every spin-wait
  int32_t* item_counter;  // next work item to hand out (zeroed before each launch)
  int32_t T_cache;      // rows of the cache tensors (bounds checks of debug builds)
  int32_t n_slots;      // partial slots in the workspace (bounds checks of debug builds)
  int32_t chk_shrink;   // debug builds: the checks treat every tensor as this many rows shorter
};

// CUDA-core fp32 path, d in {32, 64, 128}.
struct SimtParams {
  const WorkItem* items;
  int64_t n_items;
  const float *q, *ks, *vs, *kc, *vc;
  float* out;
  float* lse;
  float* part_o;
  float* part_lse;
  int32_t T_suf, H;
  float scale;
  int32_t T_cache, n_slots;
  uint32_t* status;
  int32_t chk_shrink;
};

struct MergeParams {
  const MergeJob* jobs;
  int64_t n_jobs;
  const float* part_o;
  const float* part_lse;
  void* out;
  float* lse;
  int32_t T_suf, H;
  int32_t n_slots;
  uint32_t* status;
  int32_t chk_shrink;
};

constexpr int kPackBatch = 128;
struct PackBatch {
  int64_t src_byte[kPackBatch];
  int64_t dst_byte[kPackBatch];
  int64_t bytes[kPackBatch];
  int32_t n;
  int32_t pad;
};

// Each launcher returns the cudaError_t of the launch.
cudaError_t launch_attn_tc(int d, const TcParams& p, int grid, cudaStream_t s);
size_t attn_tc_smem_bytes(int d);
constexpr int kTcThreads = 384;   // 3 warpgroups: softmax A, softmax B, control
cudaError_t launch_attn_simt(int d, const SimtParams& p, cudaStream_t s);
cudaError_t launch_merge(int d, bool out_bf16, const MergeParams& p, cudaStream_t s);
cudaError_t launch_pack(const void* ks, const void* vs, void* kc, void* vc, const PackBatch& b,
                        int64_t max_bytes, cudaStream_t s);
// Address of this device's status words [4] (word 0: status bits; 1, 2: first failed debug
// check and its value).
cudaError_t device_status_word(uint32_t** out);

}  // namespace bat
