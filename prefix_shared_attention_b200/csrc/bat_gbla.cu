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
// Three kernels; the two that stream the tokens are pipelined alike.  One CTA per SM: a
// producer warp loads 128-token tiles (plus the 8 rows before them, for the convolution) into
// a two-stage ring with TMA; eight consumer warps read them from shared memory, apply the
// convolution, feature map and gate in fp32 registers, write bf16 operand tiles in the 128-byte-
// swizzled layout, and one elected thread issues the tile's tcgen05.mma.  The next tiles' loads
// are in flight while a tile is computed.
//   gbla_state_kernel   per chunk (consecutive tiles of one (sequence, head)):
//                       D[d x d] += (w phi(k~))^T v~ (M = d, N = d, K = tokens; both operands
//                       MN-major); the partial state and n go to the workspace.
//   gbla_reduce_kernel  sums the chunks' partials of each (sequence, head) into S (bf16) and n.
//   gbla_out_kernel     per chunk: S into shared memory once; per tile phi(q~) (K-major) and
//                       O = phi(q~) . S into TMEM; the epilogue (one thread per token row) divides
//                       by n . phi(q~), normalises and gates with z (loaded by TMA beside q), writes
//                       y over z in shared memory and stores it with bulk tensor stores.
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

constexpr int kConsumerWarps = 16;
constexpr int kConsumers = 32 * kConsumerWarps;
constexpr int kThreads = kConsumers + 32;     // plus the producer warp (warp 16)
constexpr int kProducerWarp = kConsumerWarps;
constexpr int kRows = 128 / (kConsumers / 16);   // rows of a tile per consumer thread (16 threads per row)
constexpr int kPanel = 128 * 128;             // one 64-column panel of a 128-row bf16 tile
constexpr int kRawRows = 136;                 // a tile's 128 rows plus the 8 before them
constexpr int kRawPanel = kRawRows * 128;     // one 64-column panel of a raw (unswizzled) tile
constexpr int kStateStage = 4 * kRawPanel;    // raw k and v
constexpr int kOutStage = 2 * kRawPanel + 2 * kPanel;   // raw q, then z (128-byte swizzled)
constexpr float kEpsAttn = 1e-6f;
constexpr float kEpsNorm = 1e-6f;
constexpr uint64_t kWaitNs = 2000000000ull;

struct GblaSmem {
  float w[2][4 * 128];   // convolution taps (state: k, v; output: q)
  float vec[3][128];     // state: n partial; output: n, norm weight
  float den[2][128];     // output: n . phi(q~) of the tile, double-buffered
  float ss[4][128];      // output: partial sums of squares of each row, per 32-column block
  uint64_t raw_full[2], raw_empty[2], mma_done;
  uint32_t tmem_slot;
  int abort;
};
constexpr size_t kStateSmem = 1024 + 4 * kPanel + 2 * kStateStage + sizeof(GblaSmem);
constexpr size_t kOutSmem = 1024 + 4 * kPanel + 2 * kOutStage + sizeof(GblaSmem);
static_assert(kStateSmem <= 227 * 1024 && kOutSmem <= 227 * 1024, "shared memory budget");

// 16-byte chunk `c` (8 elements, c in 0..15) of row `r` of a 128-row bf16 tile held as two
// 64-column panels with the 128-byte swizzle (chunk index XOR row mod 8).
__device__ __forceinline__ uint32_t sw_off(int r, int c) {
  return (uint32_t)((c >> 3) * kPanel + r * 128 + (((c & 7) ^ (r & 7)) << 4));
}
// The same chunk of row `r` of a raw tile (two unswizzled 136-row panels).
__device__ __forceinline__ uint32_t raw_off(int r, int c) { return (uint32_t)((c >> 3) * kRawPanel + r * 128 + (c & 7) * 16); }

// elu(x) + 1, the exponential on the MUFU (2^(x log2 e)).
__device__ __forceinline__ float phi(float x) { return x > 0.f ? x + 1.f : ex2(x * 1.4426950408889634f); }
// sigmoid(x) = (1 + tanh(x / 2)) / 2: one MUFU operation.
__device__ __forceinline__ float sigmoidf_(float x) { return fmaf(0.5f, tanh_approx(0.5f * x), 0.5f); }

__device__ __forceinline__ void unpack8(const uint4& u, float (&f)[8]) {
  const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 t = __bfloat1622float2(b[i]);
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
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

__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr) {
  uint4 u;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(u.x), "=r"(u.y), "=r"(u.z), "=r"(u.w) : "r"(addr));
  return u;
}

// Barrier of the consumer warps (the producer warp does not take part).
__device__ __forceinline__ void consumer_sync() { asm volatile("bar.sync 1, 512;" ::: "memory"); }
// Same barrier, returning whether `ok` holds in every consumer thread.
__device__ __forceinline__ bool consumer_all(bool ok) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\tbar.red.and.pred q, 1, 512, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)ok)
      : "memory");
  return r != 0;
}

// Bounded wait on an mbarrier phase; false on timeout or when the CTA is aborting.
__device__ __forceinline__ bool wait_phase(uint64_t* bar, uint32_t parity, GblaSmem& sm, uint32_t* status) {
  if (mbar_test(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  while (!mbar_test_suspend(bar, parity, 1000000u)) {
    if (*reinterpret_cast<volatile int*>(&sm.abort)) return false;
    if (global_ns() - t0 > kWaitNs) {
      atomicOr(status, 1u);
      *reinterpret_cast<volatile int*>(&sm.abort) = 1;
      return false;
    }
  }
  return true;
}

// Bounded wait used after an abort (ignores the abort flag).
__device__ __forceinline__ void drain_phase(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = global_ns();
  while (!mbar_test(bar, parity))
    if (global_ns() - t0 > kWaitNs / 10) break;
}

// This thread's kRows rows (kRows*g .. of the tile) and 8 channels (16-byte chunk c) after the
// causal convolution of width 4, from a raw tile in shared memory whose row 8 is the tile's
// first token; rows before the sequence start count as zero.
__device__ __forceinline__ void conv_tile(uint32_t raw, const float* w, int c, int g, int64_t t0, int lo,
                                          float (&out)[kRows][8]) {
  uint4 r[kRows + 3];
#pragma unroll
  for (int i = 0; i < kRows + 3; ++i) {
    const int row = kRows * g + 5 + i;   // token t0 + kRows*g - 3 + i
    r[i] = (t0 + kRows * g - 3 + i >= lo) ? ld_shared_v4(raw + raw_off(row, c)) : make_uint4(0u, 0u, 0u, 0u);
  }
  float wt[4][8];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float4 w0 = *reinterpret_cast<const float4*>(w + j * 128 + c * 8);
    const float4 w1 = *reinterpret_cast<const float4*>(w + j * 128 + c * 8 + 4);
    wt[j][0] = w0.x, wt[j][1] = w0.y, wt[j][2] = w0.z, wt[j][3] = w0.w;
    wt[j][4] = w1.x, wt[j][5] = w1.y, wt[j][6] = w1.z, wt[j][7] = w1.w;
  }
  // Channel pairs go through the packed fp32x2 FMA.
#pragma unroll
  for (int i = 0; i < kRows; ++i)
#pragma unroll
    for (int e = 0; e < 8; ++e) out[i][e] = 0.f;
#pragma unroll
  for (int m = 0; m < kRows + 3; ++m) {
    float f[8];
    unpack8(r[m], f);
    // Raw row m feeds output rows i = m - 3 + j for taps j = 0..3.
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int i = m - 3 + j;
      if (i >= 0 && i < kRows) {
#pragma unroll
        for (int e = 0; e < 8; e += 2) ffma2v(out[i][e], out[i][e + 1], wt[j][e], wt[j][e + 1], f[e], f[e + 1]);
      }
    }
  }
}

__device__ __forceinline__ void tmem_alloc128(uint32_t* slot) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(slot)), "r"(128u)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_free128(uint32_t tmem) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(128u) : "memory");
}

// Producer warp: the chunk's tiles into the two-stage ring.  Map m's two 64-column panels go
// to offset map_off[m] of the stage, starting `rows_before[m]` rows before the tile (8 for the
// raw tiles the convolution reads, 0 for z); drains its loads if the CTA aborts.
template <int kStage>
__device__ __forceinline__ void produce(const GblaChunk& ch, GblaSmem& sm, uint8_t* ring, const CUtensorMap* const* maps,
                                        const int* rows_before, const int* map_off, int nmaps, uint32_t* status) {
  const int lane = threadIdx.x & 31;
  int issued = 0;
  for (int i = 0; i < ch.n_tiles; ++i) {
    const int s = i & 1;
    if (!wait_phase(&sm.raw_empty[s], ((i >> 1) & 1) ^ 1, sm, status)) break;
    if (lane == 0) {
      const int y0 = ch.seq_lo + (ch.tile0 + i) * 128;
      mbar_expect_tx(&sm.raw_full[s], kStage);
      for (int m = 0; m < nmaps; ++m)
#pragma unroll
        for (int pn = 0; pn < 2; ++pn)
          tma_load_2d(ring + s * kStage + map_off[m] + pn * (rows_before[m] ? kRawPanel : kPanel), maps[m],
                      ch.head * 128 + pn * 64, y0 - rows_before[m], &sm.raw_full[s]);
    }
    __syncwarp();
    ++issued;
  }
  if (issued < ch.n_tiles && lane == 0) {
    // Aborting: let the loads in flight land before the CTA releases its shared memory.
    for (int i = (issued > 2 ? issued - 2 : 0); i < issued; ++i) drain_phase(&sm.raw_full[i & 1], (i >> 1) & 1);
  }
  __syncwarp();
}

// ---------------------------------------------------------------------------------------
// State: partial S and n of one chunk.

__global__ void __launch_bounds__(kThreads, 1) gbla_state_kernel(const __grid_constant__ GblaParams p) {
  extern __shared__ uint8_t dyn[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dyn) + 1023) & ~uintptr_t(1023));
  uint8_t* A = base;                // (w phi(k~)) tile: rows = tokens, columns = d (MN-major A)
  uint8_t* B = base + 2 * kPanel;   // v~ tile: rows = tokens, columns = d (MN-major B)
  uint8_t* ring = base + 4 * kPanel;
  GblaSmem& sm = *reinterpret_cast<GblaSmem*>(ring + 2 * kStateStage);
  const GblaChunk ch = p.chunks[blockIdx.x];
  const int tid = threadIdx.x, warp = tid >> 5;
  const int c = tid & 15, g = (tid >> 4) & 31;
  const int h = ch.head, lo = ch.seq_lo, hi = ch.seq_hi, H = p.H;
  if (tid == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sm.raw_full[s], 1);
      mbar_init(&sm.raw_empty[s], kConsumerWarps);   // one arrival per consumer warp
    }
    mbar_init(&sm.mma_done, 1);
    sm.abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  for (int i = tid; i < 4 * 128; i += kThreads) {
    sm.w[0][i] = p.conv_k[h * 4 * 128 + i];
    sm.w[1][i] = p.conv_v[h * 4 * 128 + i];
  }
  if (tid < 128) sm.vec[0][tid] = 0.f;
  if (warp == 0) tmem_alloc128(&sm.tmem_slot);
  if (warp == kProducerWarp && (tid & 31) == 0) {
    prefetch_tmap(&p.tm_k);
    prefetch_tmap(&p.tm_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_slot;

  if (warp == kProducerWarp) {
    const CUtensorMap* maps[2] = {&p.tm_k, &p.tm_v};
    const int before[2] = {8, 8}, off[2] = {0, 2 * kRawPanel};
    produce<kStateStage>(ch, sm, ring, maps, before, off, 2, p.status);
  } else {
    float nacc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) nacc[e] = 0.f;
    const __nv_bfloat16* ax = reinterpret_cast<const __nv_bfloat16*>(p.a);
    constexpr uint32_t idesc = make_idesc(128, 128, true, true);
    bool ok = true;
    int done = 0;
    // Gate logits of this thread's rows, loaded one tile ahead (they come from global memory).
    auto load_gates = [&](int tile, __nv_bfloat16 (&a)[kRows]) {
      const int64_t tb = (int64_t)lo + (int64_t)(ch.tile0 + tile) * 128 + kRows * g;
#pragma unroll
      for (int r = 0; r < kRows; ++r) a[r] = (tile < ch.n_tiles && tb + r < hi) ? ax[(tb + r) * H + h] : __float2bfloat16(0.f);
    };
    __nv_bfloat16 a_next[kRows];
    load_gates(0, a_next);
    for (int i = 0; i < ch.n_tiles; ++i) {
      const int64_t t0 = (int64_t)lo + (int64_t)(ch.tile0 + i) * 128;
      const int s = i & 1;
      const uint32_t raw = smem_u32(ring + s * kStateStage);
      float gate[kRows];
#pragma unroll
      for (int r = 0; r < kRows; ++r) gate[r] = t0 + kRows * g + r < hi ? sigmoidf_(__bfloat162float(a_next[r])) : 0.f;
      load_gates(i + 1, a_next);
      ok = wait_phase(&sm.raw_full[s], (i >> 1) & 1, sm, p.status);
      // The previous tile's MMAs must have read the operand tiles before they are rewritten.
      if (ok && i > 0) ok = wait_phase(&sm.mma_done, (i - 1) & 1, sm, p.status);
      if (!consumer_all(ok)) {
        ok = false;
        break;
      }
      {
        float x[kRows][8];
        conv_tile(raw, sm.w[0], c, g, t0, lo, x);
#pragma unroll
        for (int r = 0; r < kRows; ++r) {
#pragma unroll
          for (int e = 0; e < 8; ++e) x[r][e] = gate[r] * phi(x[r][e]);
          const uint4 u = pack8(x[r]);
          st_shared_v4(smem_u32(A) + sw_off(kRows * g + r, c), u.x, u.y, u.z, u.w);
          float kb[8];
          unpack8(u, kb);   // n sums exactly the bf16 values the tensor core multiplies
#pragma unroll
          for (int e = 0; e < 8; ++e) nacc[e] += kb[e];
        }
      }
      {
        float x[kRows][8];
        conv_tile(raw + 2 * kRawPanel, sm.w[1], c, g, t0, lo, x);
#pragma unroll
        for (int r = 0; r < kRows; ++r) {
          const uint4 u = pack8(x[r]);
          st_shared_v4(smem_u32(B) + sw_off(kRows * g + r, c), u.x, u.y, u.z, u.w);
        }
      }
      __syncwarp();
      if ((tid & 31) == 0) mbar_arrive(&sm.raw_empty[s]);   // this warp is done with the raw tile
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      consumer_sync();
      if (warp == 0) {
        tc_fence_after();
        const uint64_t ad = sdesc_sw128(smem_u32(A), kPanel, 1024), bd = sdesc_sw128(smem_u32(B), kPanel, 1024);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)   // 16 tokens per step: two 8-row swizzle groups (2 KiB)
          mma_ss_w(tmem, ad + (uint64_t)(kk * 2048 / 16), bd + (uint64_t)(kk * 2048 / 16), idesc,
                   (i > 0 || kk > 0) ? 1u : 0u);
        tc_commit_w(&sm.mma_done);
      }
      done = i + 1;
    }
    // Partial n: this thread's 8 channels summed over its rows, then over the 16 row groups.
#pragma unroll
    for (int e = 0; e < 8; ++e) atomicAdd(&sm.vec[0][c * 8 + e], nacc[e]);
    if (done > 0) {
      if (ok) ok = wait_phase(&sm.mma_done, (done - 1) & 1, sm, p.status);
      else drain_phase(&sm.mma_done, (done - 1) & 1);
    }
    ok = consumer_all(ok);
    tc_fence_after();
    float* part = p.part_s + (int64_t)blockIdx.x * (128 * 128 + 128);
    {
      // Row i = 32 * (warp % 4) + lane of the partial state (channel i of phi(k~)), columns
      // 32 * (warp / 4) .. +31 (v channels): one 32-column TMEM load per warp.
      const int qd = warp & 3, cb = warp >> 2;
      const int i = 32 * qd + (tid & 31);
      float4* dst = reinterpret_cast<float4*>(part + (int64_t)i * 128 + 32 * cb);
      uint32_t r[32];
      tmem_ld32(tmem + ((uint32_t)(32 * qd) << 16) + 32 * cb, r);
#pragma unroll
      for (int e = 0; e < 8; ++e)
        dst[e] = (ok && done > 0) ? make_float4(__uint_as_float(r[4 * e]), __uint_as_float(r[4 * e + 1]),
                                                __uint_as_float(r[4 * e + 2]), __uint_as_float(r[4 * e + 3]))
                                  : make_float4(0.f, 0.f, 0.f, 0.f);
      if (tid < 128) part[128 * 128 + tid] = sm.vec[0][tid];
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_free128(tmem);
}

// ---------------------------------------------------------------------------------------
// Reduce: S (bf16, row-major [d][d]) and n (fp32) of each (sequence, head).

__global__ void __launch_bounds__(256) gbla_reduce_kernel(const __grid_constant__ GblaParams p) {
  // Grid (pairs, ceil((128 * 128 + 128) / 256)): one element of one pair per thread.
  const GblaPair pr = p.pairs[blockIdx.x];
  const int idx = blockIdx.y * blockDim.x + threadIdx.x;
  if (idx >= 128 * 128 + 128) return;
  float s = 0.f;
  for (int k = 0; k < pr.n_chunks; ++k) s += p.part_s[(int64_t)(pr.chunk0 + k) * (128 * 128 + 128) + idx];
  if (idx < 128 * 128)
    p.state[(int64_t)blockIdx.x * 128 * 128 + idx] = __float2bfloat16_rn(s);
  else
    p.norm_n[(int64_t)blockIdx.x * 128 + (idx - 128 * 128)] = s;
}

// ---------------------------------------------------------------------------------------
// Output: y for every token of one chunk.

__global__ void __launch_bounds__(kThreads, 1) gbla_out_kernel(const __grid_constant__ GblaParams p) {
  extern __shared__ uint8_t dyn[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dyn) + 1023) & ~uintptr_t(1023));
  uint8_t* A = base;                 // phi(q~) tile: rows = tokens, columns = d (K-major A)
  uint8_t* Bs = base + 2 * kPanel;   // S: rows = phi channels (K), columns = v channels (MN-major B)
  uint8_t* ring = base + 4 * kPanel;
  GblaSmem& sm = *reinterpret_cast<GblaSmem*>(ring + 2 * kOutStage);
  float* nvec = sm.vec[0];
  float* gw = sm.vec[1];
  const GblaChunk ch = p.chunks[blockIdx.x];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int c = tid & 15, g = (tid >> 4) & 31;
  const int h = ch.head, lo = ch.seq_lo, hi = ch.seq_hi, H = p.H;
  if (tid == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sm.raw_full[s], 1);
      mbar_init(&sm.raw_empty[s], kConsumerWarps);
    }
    mbar_init(&sm.mma_done, 1);
    sm.abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) tmem_alloc128(&sm.tmem_slot);
  if (warp == kProducerWarp && lane == 0) {
    prefetch_tmap(&p.tm_q);
    prefetch_tmap(&p.tm_z);
    prefetch_tmap(&p.tm_y);
  }
  if (warp < kConsumerWarps) {
    // S of this (sequence, head) into the B tile (row i, 16-byte chunk c of its 128 columns).
    const uint4* src = reinterpret_cast<const uint4*>(p.state + (int64_t)ch.pair * 128 * 128);
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
      const int row = kRows * g + r;
      const uint4 u = src[row * 16 + c];
      st_shared_v4(smem_u32(Bs) + sw_off(row, c), u.x, u.y, u.z, u.w);
    }
  }
  for (int i = tid; i < 4 * 128; i += kThreads) sm.w[0][i] = p.conv_q[h * 4 * 128 + i];
  if (tid < 128) {
    nvec[tid] = p.norm_n[(int64_t)ch.pair * 128 + tid];
    gw[tid] = p.norm_w[h * 128 + tid];
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_slot;

  if (warp == kProducerWarp) {
    const CUtensorMap* maps[2] = {&p.tm_q, &p.tm_z};
    const int before[2] = {8, 0}, off[2] = {0, 2 * kRawPanel};
    produce<kOutStage>(ch, sm, ring, maps, before, off, 2, p.status);
  } else {
    float nv[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) nv[e] = nvec[c * 8 + e];
    __nv_bfloat16* yx = reinterpret_cast<__nv_bfloat16*>(p.y);
    constexpr uint32_t idesc = make_idesc(128, 128, true);
    // Epilogue roles: warp w reads the TMEM rows of its lane quarter qd = w % 4 (rows 32 qd ..
    // 32 qd + 31) and the 32 columns of block cb = w / 4.
    const int qd = warp & 3, cb = warp >> 2;
    const int r = 32 * qd + lane;
    bool ok = true, stores_pending = false;
    int done = 0;
    for (int i = 0; i < ch.n_tiles; ++i) {
      const int64_t t0 = (int64_t)lo + (int64_t)(ch.tile0 + i) * 128;
      const int s = i & 1;
      const uint32_t stage = smem_u32(ring + s * kOutStage);
      float* den = sm.den[s];
      ok = wait_phase(&sm.raw_full[s], (i >> 1) & 1, sm, p.status);
      if (!consumer_all(ok)) {
        ok = false;
        break;
      }
      uint4 qu[kRows];
      {
        float x[kRows][8];
        conv_tile(stage, sm.w[0], c, g, t0, lo, x);
#pragma unroll
        for (int rr = 0; rr < kRows; ++rr) {
#pragma unroll
          for (int e = 0; e < 8; ++e) x[rr][e] = phi(x[rr][e]);
          qu[rr] = pack8(x[rr]);
          float fb[8];
          unpack8(qu[rr], fb);   // the denominator uses exactly the bf16 values the tensor core reads
          float dsum = 0.f;
#pragma unroll
          for (int e = 0; e < 8; ++e) dsum += fb[e] * nv[e];
          // Sum over the 16 threads (lanes c = 0..15 of this half-warp) holding the row's chunks.
#pragma unroll
          for (int off = 8; off > 0; off >>= 1) dsum += __shfl_xor_sync(0xffffffffu, dsum, off);
          if (c == 0) den[kRows * g + rr] = dsum;
        }
      }
      // The previous tile's MMAs must have read A before it is rewritten.
      if (i > 0) ok = wait_phase(&sm.mma_done, (i - 1) & 1, sm, p.status);
      if (!consumer_all(ok)) {
        ok = false;
        break;
      }
#pragma unroll
      for (int rr = 0; rr < kRows; ++rr)
        st_shared_v4(smem_u32(A) + sw_off(kRows * g + rr, c), qu[rr].x, qu[rr].y, qu[rr].z, qu[rr].w);
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      consumer_sync();
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
      done = i + 1;
      // Epilogue, spread over every consumer warp: each row's sum of squares from its four
      // 32-column blocks, then y = o / den / rms * g * silu(z) for this warp's block, written over
      // z in the stage (rows of a quarter that lies entirely inside the sequence) or straight to
      // y with 16-byte stores (a quarter that reaches past the sequence end).
      ok = wait_phase(&sm.mma_done, i & 1, sm, p.status);
      if (!consumer_all(ok)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int64_t t = t0 + r;
      const bool live = t < hi;
      const bool whole = t0 + 32 * qd + 31 < hi;
      uint32_t v[32];
      tmem_ld32(tmem + ((uint32_t)(32 * qd) << 16) + 32 * cb, v);
      const float inv_den = 1.f / (den[r] + kEpsAttn);
      float ssp = 0.f;
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const float o = __uint_as_float(v[e]) * inv_den;
        ssp += o * o;
      }
      sm.ss[cb][r] = ssp;
      tc_fence_before();
      consumer_sync();
      const float ss = sm.ss[0][r] + sm.ss[1][r] + sm.ss[2][r] + sm.ss[3][r];
      const float scale = inv_den * rsqrtf(ss * (1.f / 128.f) + kEpsNorm);
      const uint32_t zt = stage + 2 * kRawPanel;   // z tile: two 128-byte-swizzled panels
      uint4* yrow = reinterpret_cast<uint4*>(yx + (live ? (t * H + h) * 128 : 0));
#pragma unroll
      for (int k4 = 0; k4 < 4; ++k4) {
        const int chunk = 4 * cb + k4;   // 16-byte chunk (8 columns) of the row
        const uint32_t za = zt + sw_off(r, chunk);
        float zf[8], yv[8];
        unpack8(ld_shared_v4(za), zf);
        const float4 g0 = *reinterpret_cast<const float4*>(gw + 8 * chunk);
        const float4 g1 = *reinterpret_cast<const float4*>(gw + 8 * chunk + 4);
        const float gg[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float zz = zf[e];
          yv[e] = __uint_as_float(v[8 * k4 + e]) * scale * gg[e] * (zz * sigmoidf_(zz));   // silu(z)
        }
        const uint4 yu = pack8(yv);
        if (whole) st_shared_v4(za, yu.x, yu.y, yu.z, yu.w);
        else if (live) yrow[chunk] = yu;
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      consumer_sync();
      // Warps 0..7, lane 0: one bulk tensor store per (row quarter, 64-column panel) of a quarter
      // inside the sequence; the stage is released once the stores have read it.
      if (warp < 8 && lane == 0) {
        const int sq = warp & 3, pn = warp >> 2;
        if (t0 + 32 * sq + 31 < hi) {
          tma_store_2d(&p.tm_y, ring + s * kOutStage + 2 * kRawPanel + pn * kPanel + 32 * sq * 128, h * 128 + pn * 64,
                       (int)(t0 + 32 * sq));
          bulk_commit();
          bulk_wait_read();
          stores_pending = true;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.raw_empty[s]);
    }
    if (done > 0 && !ok) drain_phase(&sm.mma_done, (done - 1) & 1);
    if (stores_pending) bulk_wait_all();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_free128(tmem);
}

}  // namespace

cudaError_t launch_gbla(const GblaParams& p, int n_chunks, int n_pairs, cudaStream_t s) {
  if (n_chunks <= 0) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(gbla_state_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kStateSmem);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(gbla_out_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kOutSmem);
  if (e != cudaSuccess) return e;
  gbla_state_kernel<<<n_chunks, kThreads, kStateSmem, s>>>(p);
  gbla_reduce_kernel<<<dim3(n_pairs, (128 * 128 + 128 + 255) / 256), 256, 0, s>>>(p);
  gbla_out_kernel<<<n_chunks, kThreads, kOutSmem, s>>>(p);
  return cudaGetLastError();
}

}  // namespace bat
