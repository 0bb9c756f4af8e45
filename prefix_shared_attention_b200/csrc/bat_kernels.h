// Kernel parameter blocks and host-side launchers (internal to libbat.so).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include "bat_internal.h"

namespace bat {

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
  uint32_t* status;     // device status word (bit 0: a wait timed out)
  uint64_t wait_ns;     // bound on every spin-wait
  int32_t* item_counter;  // next work item to hand out (zeroed before each launch)
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
};

struct MergeParams {
  const MergeJob* jobs;
  int64_t n_jobs;
  const float* part_o;
  const float* part_lse;
  void* out;
  float* lse;
  int32_t T_suf, H;
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
// Address of this device's status word (resolved once per device).
cudaError_t device_status_word(uint32_t** out);

}  // namespace bat
