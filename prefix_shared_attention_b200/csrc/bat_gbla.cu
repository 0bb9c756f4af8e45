// Gated bidirectional linear attention (GBLA) forward on tcgen05 tensor cores (sm_100a).
//
// Operation ("Gated Bidirectional Linear Attention for Generative Retrieval", sections
// "Abstract" and the summary above it): kernelized linear attention with no mask over each
// user history, extended by a local causal convolution of q, k and v, a per-token key gate
// that softly forgets tokens, and a gated RMSNorm output.  Per sequence and head (d = 128):
//
//   x~[t] = sum_{j<4} c_x[j] * x[t-j]  (zero before the sequence start; x in q, k, v)
//   S = sum_t sigmoid(a[t]) phi(k~[t]) v~[t]^T,   n = sum_t sigmoid(a[t]) phi(k~[t])
//   o[t] = S^T phi(q~[t]) / (n . phi(q~[t]) + 1e-6),   phi(x) = elu(x) + 1
//   y[t] = o[t] / sqrt(mean(o[t]^2) + 1e-6) * g * silu(z[t])
//
// Three kernels, each one pass over its tokens:
//   gbla_state_kernel   per chunk of 128-token tiles of one (sequence, head): the threads
//                       read k, v and the gate logits (16-byte coalesced loads), apply the
//                       convolution, phi and the gate in registers and write bf16 operand tiles
//                       to shared memory in the 128-byte-swizzled layout; one thread issues
//                       tcgen05.mma D[d x d] += (w phi(k~))^T v~ (M = d, N = d, K = tokens, both
//                       operands MN-major); the partial state and partial n go to the workspace.
//   gbla_reduce_kernel  sums the chunks' partials of each (sequence, head) into S (bf16) and n.
//   gbla_out_kernel     per chunk: S into shared memory once, then per tile phi(q~) (K-major
//                       operand) and tcgen05.mma O = phi(q~) . S into TMEM; the epilogue (one
//                       thread per token row) divides by n . phi(q~), normalises and gates.
// The path is HBM-bound (about 0.4 d FLOP per byte): q, k, v, z and the gate logits are read
// once and y is written once; S and the partials stay small and in L2.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "bat_gbla_internal.h"
#include "bat_kernels.h"

namespace bat {
namespace {

#include "bat_ptx.h"

constexpr int kThreads = 256;
constexpr int kPanel = 128 * 128;   // bytes of one 64-column panel of a 128-row bf16 tile
constexpr float kEpsAttn = 1e-6f;
constexpr float kEpsNorm = 1e-6f;
constexpr uint64_t kWaitNs = 2000000000ull;

// 16-byte chunk `c` (8 elements, c in 0..15) of row `r` of a 128 x 128 bf16 tile held as two
// 64-column panels with the 128-byte swizzle (chunk index XOR row mod 8).
__device__ __forceinline__ uint32_t sw_off(int r, int c) {
  return (uint32_t)((c >> 3) * kPanel + r * 128 + (((c & 7) ^ (r & 7)) << 4));
}

__device__ __forceinline__ float phi(float x) { return x > 0.f ? x + 1.f : __expf(x); }
__device__ __forceinline__ float sigmoidf_(float x) { return 1.f / (1.f + __expf(-x)); }

__device__ __forceinline__ void unpack8(const uint4& u, float (&f)[8]) {
  const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 t = __bfloat1622float2(b[i]);
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}

// Bounded wait on an mbarrier phase (every thread of the CTA may call it); false on timeout.
__device__ __forceinline__ bool wait_phase(uint64_t* bar, uint32_t parity, uint32_t* status) {
  if (mbar_test(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  while (!mbar_test_suspend(bar, parity, 1000000u)) {
    if (global_ns() - t0 > kWaitNs) {
      atomicOr(status, 1u);
      return false;
    }
  }
  return true;
}

// Loads this thread's 16-byte chunk `c` of rows t0+8g-3 .. t0+8g+7 of x (token-major [T, H, 128]
// bf16, head h), with zero for rows outside [lo, hi): the 3 rows before its 8 rows feed the
// convolution.
__device__ __forceinline__ void load_rows(const __nv_bfloat16* x, int64_t t_first, int lo, int hi, int H, int h, int c,
                                          uint4 (&r)[11]) {
#pragma unroll
  for (int i = 0; i < 11; ++i) {
    const int64_t t = t_first + i;
    r[i] = (t >= lo && t < hi)
               ? __ldg(reinterpret_cast<const uint4*>(x + (t * H + h) * 128) + c)
               : make_uint4(0u, 0u, 0u, 0u);
  }
}

// Depthwise causal convolution of width 4, row i (0..7) of this thread's 8 rows and 8 channels:
// out[e] = sum_j w[j][c*8+e] * in[i + 3 - j][e], with w (4 x 128 fp32) in shared memory.
__device__ __forceinline__ void conv_row(const uint4 (&raw)[11], const float* w, int c, int i, float (&out)[8]) {
#pragma unroll
  for (int e = 0; e < 8; ++e) out[e] = 0.f;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    float f[8];
    unpack8(raw[i + 3 - j], f);
    const float4 w0 = *reinterpret_cast<const float4*>(w + j * 128 + c * 8);
    const float4 w1 = *reinterpret_cast<const float4*>(w + j * 128 + c * 8 + 4);
    out[0] += w0.x * f[0];
    out[1] += w0.y * f[1];
    out[2] += w0.z * f[2];
    out[3] += w0.w * f[3];
    out[4] += w1.x * f[4];
    out[5] += w1.y * f[5];
    out[6] += w1.z * f[6];
    out[7] += w1.w * f[7];
  }
}

__device__ __forceinline__ uint4 pack8(const float (&v)[8]) {
  uint4 u;
  u.x = pack_bf16x2(v[0], v[1]);
  u.y = pack_bf16x2(v[2], v[3]);
  u.z = pack_bf16x2(v[4], v[5]);
  u.w = pack_bf16x2(v[6], v[7]);
  return u;
}

__device__ __forceinline__ void round8(const uint4& u, float (&v)[8]) { unpack8(u, v); }

// Dynamic shared memory of both kernels: two 128 x 128 bf16 operand tiles (1 KiB aligned for
// the 128-byte swizzle), then small per-CTA arrays.
constexpr size_t kTilesBytes = 4 * kPanel;
struct GblaSmem {
  float w[2][4 * 128];   // convolution weights (state: k, v; output: q)
  float vec[3][128];     // state: n partial; output: n, denominators, norm weight
  uint64_t mma_done;
  uint32_t tmem_slot;
};
constexpr size_t kSmemBytes = 1024 + kTilesBytes + sizeof(GblaSmem);

// ---------------------------------------------------------------------------------------
// State: partial S and n of one chunk.

__global__ void __launch_bounds__(kThreads, 2) gbla_state_kernel(const GblaParams p) {
  extern __shared__ uint8_t dyn[];
  uint8_t* tiles = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dyn) + 1023) & ~uintptr_t(1023));
  uint8_t* A = tiles;               // (w phi(k~)) tile: rows = tokens, columns = d (MN-major A)
  uint8_t* B = tiles + 2 * kPanel;  // v~ tile: rows = tokens, columns = d (MN-major B)
  GblaSmem& sm = *reinterpret_cast<GblaSmem*>(tiles + kTilesBytes);
  const GblaChunk ch = p.chunks[blockIdx.x];
  const int tid = threadIdx.x, warp = tid >> 5;
  const int c = tid & 15, g = tid >> 4;
  const int h = ch.head, lo = ch.seq_lo, hi = ch.seq_hi, H = p.H;
  if (tid == 0) {
    mbar_init(&sm.mma_done, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  for (int i = tid; i < 4 * 128; i += kThreads) {
    sm.w[0][i] = p.conv_k[h * 4 * 128 + i];
    sm.w[1][i] = p.conv_v[h * 4 * 128 + i];
  }
  if (tid < 128) sm.vec[0][tid] = 0.f;
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&sm.tmem_slot)),
                 "r"(128u)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_slot;
  float nacc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) nacc[e] = 0.f;
  const __nv_bfloat16* kx = reinterpret_cast<const __nv_bfloat16*>(p.k);
  const __nv_bfloat16* vx = reinterpret_cast<const __nv_bfloat16*>(p.v);
  const __nv_bfloat16* ax = reinterpret_cast<const __nv_bfloat16*>(p.a);
  constexpr uint32_t idesc = make_idesc(128, 128, true, true);
  bool ok = true;
  for (int tile = 0; tile < ch.n_tiles; ++tile) {
    const int64_t t0 = (int64_t)lo + (int64_t)(ch.tile0 + tile) * 128;
    uint4 raw[11];
    load_rows(kx, t0 + 8 * g - 3, lo, hi, H, h, c, raw);
    float gate[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int64_t t = t0 + 8 * g + i;
      gate[i] = t < hi ? sigmoidf_(__bfloat162float(ax[t * H + h])) : 0.f;
    }
    // The previous tile's MMAs must have read the operand tiles before they are rewritten
    // (one decision for the whole CTA).
    if (tile > 0) ok = wait_phase(&sm.mma_done, (tile - 1) & 1, p.status);
    if (!__syncthreads_and(ok)) {
      ok = false;
      break;
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      float kc[8];
      conv_row(raw, sm.w[0], c, i, kc);
#pragma unroll
      for (int e = 0; e < 8; ++e) kc[e] = gate[i] * phi(kc[e]);
      const uint4 u = pack8(kc);
      round8(u, kc);   // n sums exactly the bf16 values the tensor core multiplies
#pragma unroll
      for (int e = 0; e < 8; ++e) nacc[e] += kc[e];
      st_shared_v4(smem_u32(A) + sw_off(8 * g + i, c), u.x, u.y, u.z, u.w);
    }
    load_rows(vx, t0 + 8 * g - 3, lo, hi, H, h, c, raw);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      float vc[8];
      conv_row(raw, sm.w[1], c, i, vc);
      const uint4 u = pack8(vc);
      st_shared_v4(smem_u32(B) + sw_off(8 * g + i, c), u.x, u.y, u.z, u.w);
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncthreads();
    if (warp == 0) {
      tc_fence_after();
      const uint64_t ad = sdesc_sw128(smem_u32(A), kPanel, 1024), bd = sdesc_sw128(smem_u32(B), kPanel, 1024);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)   // 16 tokens per step: two 8-row swizzle groups (2 KiB)
        mma_ss_w(tmem, ad + (uint64_t)(kk * 2048 / 16), bd + (uint64_t)(kk * 2048 / 16), idesc,
                 (tile > 0 || kk > 0) ? 1u : 0u);
      tc_commit_w(&sm.mma_done);
    }
  }
  // Partial n: this thread's 8 channels summed over its rows, then over the 16 row groups.
#pragma unroll
  for (int e = 0; e < 8; ++e) atomicAdd(&sm.vec[0][c * 8 + e], nacc[e]);
  if (ok && ch.n_tiles > 0) ok = wait_phase(&sm.mma_done, (ch.n_tiles - 1) & 1, p.status);
  ok = __syncthreads_and(ok);
  tc_fence_after();
  float* part = p.part_s + (int64_t)blockIdx.x * (128 * 128 + 128);
  if (warp < 4) {
    // Row i = 32 * warp + lane of the partial state: channel i of phi(k~), all 128 v channels.
    const int i = 32 * warp + (tid & 31);
    float4* dst = reinterpret_cast<float4*>(part + (int64_t)i * 128);
#pragma unroll 1
    for (int q = 0; q < 4; ++q) {
      uint32_t r[32];
      tmem_ld32(tmem + ((uint32_t)(32 * warp) << 16) + 32 * q, r);
#pragma unroll
      for (int e = 0; e < 8; ++e)
        dst[8 * q + e] = ok ? make_float4(__uint_as_float(r[4 * e]), __uint_as_float(r[4 * e + 1]),
                                          __uint_as_float(r[4 * e + 2]), __uint_as_float(r[4 * e + 3]))
                            : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  } else if (tid >= 128) {
    part[128 * 128 + (tid - 128)] = sm.vec[0][tid - 128];
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(128u) : "memory");
}

// ---------------------------------------------------------------------------------------
// Reduce: S (bf16, row-major [d][d]) and n (fp32) of each (sequence, head).

__global__ void __launch_bounds__(256) gbla_reduce_kernel(const GblaParams p) {
  const GblaPair pr = p.pairs[blockIdx.x];
  for (int idx = threadIdx.x; idx < 128 * 128 + 128; idx += blockDim.x) {
    float s = 0.f;
    for (int k = 0; k < pr.n_chunks; ++k) s += p.part_s[(int64_t)(pr.chunk0 + k) * (128 * 128 + 128) + idx];
    if (idx < 128 * 128)
      p.state[(int64_t)blockIdx.x * 128 * 128 + idx] = __float2bfloat16_rn(s);
    else
      p.norm_n[(int64_t)blockIdx.x * 128 + (idx - 128 * 128)] = s;
  }
}

// ---------------------------------------------------------------------------------------
// Output: y for every token of one chunk.

__global__ void __launch_bounds__(kThreads, 2) gbla_out_kernel(const GblaParams p) {
  extern __shared__ uint8_t dyn[];
  uint8_t* tiles = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dyn) + 1023) & ~uintptr_t(1023));
  uint8_t* A = tiles;                // phi(q~) tile: rows = tokens, columns = d (K-major A)
  uint8_t* Bs = tiles + 2 * kPanel;  // S: rows = phi channels (K), columns = v channels (MN-major B)
  GblaSmem& sm = *reinterpret_cast<GblaSmem*>(tiles + kTilesBytes);
  float* nvec = sm.vec[0];
  float* den = sm.vec[1];
  float* gw = sm.vec[2];
  const GblaChunk ch = p.chunks[blockIdx.x];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int c = tid & 15, g = tid >> 4;
  const int h = ch.head, lo = ch.seq_lo, hi = ch.seq_hi, H = p.H;
  if (tid == 0) {
    mbar_init(&sm.mma_done, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&sm.tmem_slot)),
                 "r"(128u)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  // S of this (sequence, head) into the B tile (row i, 16-byte chunk c of its 128 columns), the
  // convolution weights of q, n and the norm weight.
  {
    const uint4* src = reinterpret_cast<const uint4*>(p.state + (int64_t)ch.pair * 128 * 128);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int r = 8 * g + i;
      const uint4 u = src[r * 16 + c];
      st_shared_v4(smem_u32(Bs) + sw_off(r, c), u.x, u.y, u.z, u.w);
    }
    for (int i = tid; i < 4 * 128; i += kThreads) sm.w[0][i] = p.conv_q[h * 4 * 128 + i];
    if (tid < 128) {
      nvec[tid] = p.norm_n[(int64_t)ch.pair * 128 + tid];
      gw[tid] = p.norm_w[h * 128 + tid];
    }
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_slot;
  float nv[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) nv[e] = nvec[c * 8 + e];
  const __nv_bfloat16* qx = reinterpret_cast<const __nv_bfloat16*>(p.q);
  const __nv_bfloat16* zx = reinterpret_cast<const __nv_bfloat16*>(p.z);
  __nv_bfloat16* yx = reinterpret_cast<__nv_bfloat16*>(p.y);
  constexpr uint32_t idesc = make_idesc(128, 128, true);
  for (int tile = 0; tile < ch.n_tiles; ++tile) {
    const int64_t t0 = (int64_t)lo + (int64_t)(ch.tile0 + tile) * 128;
    uint4 raw[11];
    load_rows(qx, t0 + 8 * g - 3, lo, hi, H, h, c, raw);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      float f[8];
      conv_row(raw, sm.w[0], c, i, f);
#pragma unroll
      for (int e = 0; e < 8; ++e) f[e] = phi(f[e]);
      const uint4 u = pack8(f);
      round8(u, f);   // the denominator uses exactly the bf16 values the tensor core reads
      float dsum = 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) dsum += f[e] * nv[e];
      // Sum over the 16 threads (lanes c = 0..15 of this half-warp) holding the row's chunks.
#pragma unroll
      for (int off = 8; off > 0; off >>= 1) dsum += __shfl_xor_sync(0xffffffffu, dsum, off);
      const int r = 8 * g + i;
      if (c == 0) den[r] = dsum;
      st_shared_v4(smem_u32(A) + sw_off(r, c), u.x, u.y, u.z, u.w);
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncthreads();
    if (warp == 0) {
      tc_fence_after();
      const uint64_t ad = sdesc_sw128(smem_u32(A), 16, 1024), bd = sdesc_sw128(smem_u32(Bs), kPanel, 1024);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {   // 16 channels per step
        const uint64_t aoff = (uint64_t)(((kk >> 2) * kPanel + (kk & 3) * 32) >> 4);
        mma_ss_w(tmem, ad + aoff, bd + (uint64_t)(kk * 2048 / 16), idesc, kk > 0 ? 1u : 0u);
      }
      tc_commit_w(&sm.mma_done);
    }
    if (!__syncthreads_and(wait_phase(&sm.mma_done, tile & 1, p.status))) break;
    tc_fence_after();
    if (warp < 4) {
      // Epilogue: thread = token row (TMEM lane).
      const int r = 32 * warp + lane;
      const int64_t t = t0 + r;
      const uint32_t trow = tmem + ((uint32_t)(32 * warp) << 16);
      const float inv_den = 1.f / (den[r] + kEpsAttn);
      float ss = 0.f;
#pragma unroll 1
      for (int q = 0; q < 4; ++q) {
        uint32_t v[32];
        tmem_ld32(trow + 32 * q, v);
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const float o = __uint_as_float(v[e]) * inv_den;
          ss += o * o;
        }
      }
      const float scale = inv_den * rsqrtf(ss * (1.f / 128.f) + kEpsNorm);
      // Every lane takes part in the TMEM loads (tcgen05.ld is warp-collective); only rows of
      // the sequence read z and store y.
      const bool live = t < hi;
      const int64_t trow_g = live ? (t * H + h) * 128 : 0;
      const uint4* zr = reinterpret_cast<const uint4*>(zx + trow_g);
      uint4* yr = reinterpret_cast<uint4*>(yx + trow_g);
#pragma unroll 1
      for (int q = 0; q < 4; ++q) {
        uint32_t v[32];
        tmem_ld32(trow + 32 * q, v);
        if (live) {
#pragma unroll
          for (int k4 = 0; k4 < 4; ++k4) {
            float zf[8], yv[8];
            unpack8(__ldg(zr + 4 * q + k4), zf);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const float zz = zf[e];
              yv[e] = __uint_as_float(v[8 * k4 + e]) * scale * gw[32 * q + 8 * k4 + e] * (zz / (1.f + __expf(-zz)));
            }
            yr[4 * q + k4] = pack8(yv);
          }
        }
      }
    }
    tc_fence_before();
    __syncthreads();   // the MMA has read A and the epilogue has read TMEM before the next tile
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(128u) : "memory");
}

}  // namespace

cudaError_t launch_gbla(const GblaParams& p, int n_chunks, int n_pairs, cudaStream_t s) {
  if (n_chunks <= 0) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(gbla_state_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(gbla_out_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  gbla_state_kernel<<<n_chunks, kThreads, kSmemBytes, s>>>(p);
  gbla_reduce_kernel<<<n_pairs, 256, 0, s>>>(p);
  gbla_out_kernel<<<n_chunks, kThreads, kSmemBytes, s>>>(p);
  return cudaGetLastError();
}

}  // namespace bat
