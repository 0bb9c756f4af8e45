// Internal definitions of the GBLA path (gated bidirectional linear attention): the work list
// of the three kernels and their parameter block.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

namespace bat {

// A chunk: consecutive 128-token tiles of one (sequence, head).  The state kernel computes the
// chunk's partial state, the output kernel the chunk's outputs.
struct GblaChunk {
  int32_t pair;     // index of the (sequence, head) pair
  int32_t head;
  int32_t seq_lo;   // first token of the sequence
  int32_t seq_hi;   // one past its last token
  int32_t tile0;    // first tile of the chunk (128 tokens each, from seq_lo)
  int32_t n_tiles;
  int32_t pad0, pad1;
};
static_assert(sizeof(GblaChunk) == 32, "GblaChunk is 32 bytes");

// The chunks of one (sequence, head) pair are consecutive in the chunk list.
struct GblaPair {
  int32_t chunk0, n_chunks;
};

struct alignas(64) GblaParams {
  // 2-D tensor maps over [T, H * 128] bf16: q, k, v with a box of 64 columns x 136 rows (a tile
  // and the 8 rows before it) and no swizzle (the threads read them); z with a box of 64 x 128
  // and y (bulk stores) with 64 x 32, both with the 128-byte swizzle.
  CUtensorMap tm_q, tm_k, tm_v, tm_z, tm_y;
  const GblaChunk* chunks;
  const GblaPair* pairs;
  const void *q, *k, *v;    // bf16 [T, H, 128]
  const void* a;            // bf16 [T, H] key-gate logits
  const void* z;            // bf16 [T, H, 128] output gate
  const float *conv_q, *conv_k, *conv_v;   // fp32 [H, 4, 128]
  const float* norm_w;      // fp32 [H, 128]
  void* y;                  // bf16 [T, H, 128]
  float* part_s;            // workspace: per chunk [128 x 128] partial state then [128] partial n
  __nv_bfloat16* state;     // workspace: per pair [128 x 128] bf16 state (row i = phi channel)
  float* norm_n;            // workspace: per pair [128] n
  int32_t H;
  int32_t pad;
  uint32_t* status;         // device status word (bit 0: a wait timed out)
  uint64_t wait_ns;         // bound on every spin-wait (bat_set_wait_timeout_ns)
};

cudaError_t launch_gbla(const GblaParams& p, int n_chunks, int n_pairs, cudaStream_t s);
uint64_t wait_limit_ns();   // the current bat_set_wait_timeout_ns setting

}  // namespace bat
