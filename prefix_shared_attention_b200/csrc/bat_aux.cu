// Companion kernels of the attention forward:
//   * the fp32 path (CUDA cores, exact fp32 softmax) for fp32 tensors, d in {32, 64, 128};
//   * the log-sum-exp merge of split query tiles (Bat lead page, section "This paper's
//     idea": either block may be the prefix because softmax over a union of key sets is
//     the weighted combination of the softmaxes over its parts);
//   * the prefix K/V pack into the cache pool (section "Problem": the shared prefix's K/V
//     is computed once and kept for reuse).
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "bat_kernels.h"

namespace bat {
namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.69314718055994531f;

// One warp per query row; each lane holds D/32 contiguous elements of q and of the output.
// Scores are reduced across the warp with butterfly shuffles.
template <int D>
__global__ void __launch_bounds__(128) bat_attn_simt_kernel(const SimtParams p) {
  constexpr int E = D / 32;
  const WorkItem w = p.items[blockIdx.x];
  const int X = blockIdx.y;
  if (X >= w.n_q) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rows = X ? w.qB_rows : w.qA_rows;
  const int q0 = X ? w.qB_row0 : w.qA_row0;
  const bool own_a = w.shared || X == 0 || w.n_q == 1;
  const int s_row0 = own_a ? w.sA_row0 : w.sB_row0;
  const int s_len = own_a ? w.sA_len : w.sB_len;
  const int64_t row_stride = (int64_t)p.H * D;
  const int64_t col = (int64_t)w.head * D + lane * E;
  // Debug builds: every row this query tile reads or writes lies inside its tensor.
  if (!BAT_DCHECK(p.status,
                  w.head >= 0 && w.head < p.H && rows >= 0 && rows <= kTileM && q0 >= 0 && q0 + rows <= (p.T_suf - p.chk_shrink) &&
                      s_row0 >= 0 && s_row0 + s_len <= (p.T_suf - p.chk_shrink) &&
                      (w.pre_len == 0 || (w.pre_row0 >= 0 && w.pre_row0 + w.pre_len <= (p.T_cache - p.chk_shrink))) &&
                      (w.split_slot < 0 || (w.split_slot >= 0 && w.split_slot + X < p.n_slots)),
                  kChkSimtRow, blockIdx.x))
    return;
  for (int r = warp; r < rows; r += 4) {
    float q[E], o[E];
#pragma unroll
    for (int e = 0; e < E; ++e) {
      q[e] = p.q[(int64_t)(q0 + r) * row_stride + col + e];
      o[e] = 0.f;
    }
    float m = -INFINITY, l = 0.f;
    auto visit = [&](const float* K, const float* V, int64_t krow) {
      float dot = 0.f;
#pragma unroll
      for (int e = 0; e < E; ++e) dot = fmaf(q[e], K[krow * row_stride + col + e], dot);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
      const float s = dot * p.scale;
      const float m_new = fmaxf(m, s);
      const float alpha = expf(m - m_new);
      const float pe = expf(s - m_new);
      l = l * alpha + pe;
#pragma unroll
      for (int e = 0; e < E; ++e) o[e] = fmaf(o[e], alpha, pe * V[krow * row_stride + col + e]);
      m = m_new;
    };
    for (int j = 0; j < w.pre_len; ++j) visit(p.kc, p.vc, (int64_t)w.pre_row0 + j);
    for (int j = 0; j < s_len; ++j) visit(p.ks, p.vs, (int64_t)s_row0 + j);
    const float inv = 1.f / l;
    const int64_t qrow = q0 + r;
    if (w.split_slot < 0) {
#pragma unroll
      for (int e = 0; e < E; ++e) p.out[qrow * row_stride + col + e] = o[e] * inv;
      if (lane == 0 && p.lse) p.lse[(int64_t)w.head * p.T_suf + qrow] = m + logf(l);
    } else {
      const int64_t slot = w.split_slot + X;
#pragma unroll
      for (int e = 0; e < E; ++e) p.part_o[(slot * kTileM + r) * D + lane * E + e] = o[e] * inv;
      if (lane == 0) p.part_lse[slot * kTileM + r] = (m + logf(l)) * kLog2e;
    }
  }
}

template <typename OutT>
__device__ __forceinline__ void store4(OutT* dst, float a, float b, float c, float d);
template <>
__device__ __forceinline__ void store4<float>(float* dst, float a, float b, float c, float d) {
  *reinterpret_cast<float4*>(dst) = make_float4(a, b, c, d);
}
template <>
__device__ __forceinline__ void store4<__nv_bfloat16>(__nv_bfloat16* dst, float a, float b, float c, float d) {
  __nv_bfloat162 lo = __floats2bfloat162_rn(a, b), hi = __floats2bfloat162_rn(c, d);
  uint2 v;
  v.x = *reinterpret_cast<uint32_t*>(&lo);
  v.y = *reinterpret_cast<uint32_t*>(&hi);
  *reinterpret_cast<uint2*>(dst) = v;
}

// One block per split query tile: weights w_i = 2^(lse_i - max), O = sum w_i O_i / sum w_i.
template <typename OutT, int D>
__global__ void __launch_bounds__(256) bat_merge_kernel(const MergeParams p) {
  const MergeJob j = p.jobs[blockIdx.x];
  constexpr int C4 = D / 4;
  // Debug builds: every partial it reads and every row it writes lies inside its buffer.
  if (!BAT_DCHECK(p.status,
                  j.n_chunks >= 1 && j.slot0 >= 0 && j.slot_stride >= 0 &&
                      j.slot0 + (int64_t)(j.n_chunks - 1) * j.slot_stride < p.n_slots && j.q_rows >= 0 &&
                      j.q_rows <= kTileM && j.q_row0 >= 0 && j.q_row0 + j.q_rows <= (p.T_suf - p.chk_shrink) && j.head >= 0 &&
                      j.head < p.H,
                  kChkMerge, blockIdx.x))
    return;
  for (int idx = threadIdx.x; idx < j.q_rows * C4; idx += blockDim.x) {
    const int r = idx / C4, c4 = idx % C4;
    float mx = -INFINITY;
    for (int c = 0; c < j.n_chunks; ++c)
      mx = fmaxf(mx, p.part_lse[(int64_t)(j.slot0 + c * j.slot_stride) * kTileM + r]);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float tot = 0.f;
    for (int c = 0; c < j.n_chunks; ++c) {
      const int64_t slot = j.slot0 + (int64_t)c * j.slot_stride;
      const float wgt = exp2f(p.part_lse[slot * kTileM + r] - mx);
      const float4 v = *reinterpret_cast<const float4*>(p.part_o + (slot * kTileM + r) * D + 4 * c4);
      tot += wgt;
      acc.x = fmaf(wgt, v.x, acc.x);
      acc.y = fmaf(wgt, v.y, acc.y);
      acc.z = fmaf(wgt, v.z, acc.z);
      acc.w = fmaf(wgt, v.w, acc.w);
    }
    const float inv = 1.f / tot;
    const int64_t qrow = j.q_row0 + r;
    OutT* dst = reinterpret_cast<OutT*>(p.out) + (qrow * p.H + j.head) * D + 4 * c4;
    store4<OutT>(dst, acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
    if (c4 == 0 && p.lse) p.lse[(int64_t)j.head * p.T_suf + qrow] = (mx + log2f(tot)) * kLn2;
  }
}

// Batched contiguous copies: prefix i's rows are one contiguous byte range in the source
// and in the pool, both token-major [T, H, d].
__global__ void __launch_bounds__(256) bat_pack_kernel(const uint4* __restrict__ ks, const uint4* __restrict__ vs,
                                                       uint4* __restrict__ kc, uint4* __restrict__ vc,
                                                       const PackBatch b) {
  const int i = blockIdx.y;
  if (i >= b.n) return;
  const int64_t n = b.bytes[i] / 16, s = b.src_byte[i] / 16, d = b.dst_byte[i] / 16;
  for (int64_t v = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; v < n; v += (int64_t)gridDim.x * blockDim.x) {
    kc[d + v] = ks[s + v];
    vc[d + v] = vs[s + v];
  }
}

}  // namespace

cudaError_t launch_attn_simt(int d, const SimtParams& p, cudaStream_t s) {
  if (p.n_items <= 0) return cudaSuccess;
  if (p.n_items > 0x7fffffff) return cudaErrorInvalidValue;
  const dim3 grid((unsigned)p.n_items, 2);
  switch (d) {
    case 32: bat_attn_simt_kernel<32><<<grid, 128, 0, s>>>(p); break;
    case 64: bat_attn_simt_kernel<64><<<grid, 128, 0, s>>>(p); break;
    case 128: bat_attn_simt_kernel<128><<<grid, 128, 0, s>>>(p); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_merge(int d, bool out_bf16, const MergeParams& p, cudaStream_t s) {
  if (p.n_jobs <= 0) return cudaSuccess;
  if (p.n_jobs > 0x7fffffff) return cudaErrorInvalidValue;
  const unsigned g = (unsigned)p.n_jobs;
  if (out_bf16) {
    if (d == 64) bat_merge_kernel<__nv_bfloat16, 64><<<g, 256, 0, s>>>(p);
    else if (d == 128) bat_merge_kernel<__nv_bfloat16, 128><<<g, 256, 0, s>>>(p);
    else return cudaErrorInvalidValue;
  } else {
    if (d == 32) bat_merge_kernel<float, 32><<<g, 256, 0, s>>>(p);
    else if (d == 64) bat_merge_kernel<float, 64><<<g, 256, 0, s>>>(p);
    else if (d == 128) bat_merge_kernel<float, 128><<<g, 256, 0, s>>>(p);
    else return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_pack(const void* ks, const void* vs, void* kc, void* vc, const PackBatch& b, int64_t max_bytes,
                        cudaStream_t s) {
  if (b.n <= 0 || max_bytes <= 0) return cudaSuccess;
  int64_t blocks = (max_bytes / 16 + 255) / 256;
  if (blocks > 1024) blocks = 1024;
  const dim3 grid((unsigned)blocks, (unsigned)b.n);
  bat_pack_kernel<<<grid, 256, 0, s>>>(static_cast<const uint4*>(ks), static_cast<const uint4*>(vs),
                                       static_cast<uint4*>(kc), static_cast<uint4*>(vc), b);
  return cudaGetLastError();
}

}  // namespace bat
