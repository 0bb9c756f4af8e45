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
// Three kernels; the two that stream the tokens are pipelined alike.  One CTA of 16 warps per
// SM: 128-token tiles (plus the 8 rows before them, for the convolution) arrive by TMA in
// two-stage rings, issued by thread 0 right after the tile barrier that shows every warp done
// with the stage; the warps read them from shared memory (each thread 8
// consecutive rows x 4 channels, so the convolution reads 11 raw rows per 8 outputs), apply the
// convolution, feature map and gate in fp32 registers, write 16-bit operand tiles (fp16 for
// the state contraction, bf16 for the output one) in the 128-byte-swizzled layout, and one
// elected thread issues the tile's tcgen05.mma.  The next tiles' loads are in flight while a
// tile is computed.
//   gbla_state_kernel   per chunk (consecutive tiles of one (sequence, head)):
//                       D[d x (d+16)] += (w phi(k~))^T [v~ | 1] (M = d, N = d + 16, K = tokens;
//                       both operands MN-major; the ones column gives n); the partial state and
//                       n go to the workspace.
//   gbla_reduce_kernel  sums the chunks' partials of each (sequence, head) into S (bf16) and n.
//   gbla_out_kernel     per chunk: [S | n] into shared memory once; per tile phi(q~) (K-major)
//                       and [O | n . phi(q~)] = phi(q~) . [S | n] into one of two TMEM
//                       accumulators; the epilogue of the previous tile (four warps per row
//                       quarter, 32 columns each) divides by the denominator, normalises and
//                       gates with z (its own ring), writes y over z in shared memory and stores
//                       it with bulk tensor stores.
// The path is HBM-bound (about 0.4 d FLOP per byte): q, k, v, z and the gate logits are read
// once and y is written once; S and the partials stay small and in L2.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "bat_gbla_internal.h"
#include "bat_kernels.h"

namespace bat {
namespace {

#include "bat_ptx.h"

// (d0, d1) = (a0, a1) * (b0, b1) on the packed fp32x2 path.
__device__ __forceinline__ void fmul2v(float& d0, float& d1, float a0, float a1, float b0, float b1) {
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

// (d0, d1) = (a0, a1) * (b0, b1) + (c0, c1) on the packed fp32x2 FMA path.
__device__ __forceinline__ void ffma2c(float& d0, float& d1, float a0, float a1, float b0, float b1, float c0,
                                       float c1) {
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1), "f"(c0), "f"(c1));
}

__device__ __forceinline__ float lg2_approx(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

constexpr int kConsumerWarps = 16;
constexpr int kConsumers = 32 * kConsumerWarps;   // every thread of a CTA
// Consumer thread (warp w, lane l): rows 8w .. 8w+7 of a tile, channels 4l .. 4l+3.
constexpr int kRowsT = 8;
constexpr int kPanel = 128 * 128;             // one 64-column panel of a 128-row bf16 tile
constexpr int kRawRows = 136;                 // a tile's 128 rows plus the 8 before them
constexpr int kRawPanel = kRawRows * 128;     // one 64-column panel of a raw (unswizzled) tile
constexpr int kStateStage = 4 * kRawPanel;    // raw k and v
constexpr int kQStage = 2 * kRawPanel;        // raw q
constexpr int kZStage = 2 * kPanel;           // z (128-byte swizzled), then y over it
// MMA width: the 128 channels plus a third operand panel whose first column carries a ones
// column (state: n = (w phi(k~))^T 1) or n itself (output: n . phi(q~)), so the tensor core
// produces n and the denominator beside the product.
constexpr int kN = 144;
constexpr uint32_t kAccStride = 256;          // TMEM columns between the output kernel's two accumulators
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kEpsAttn = 1e-6f;
constexpr float kEpsNorm = 1e-6f;
// Upper bound on the waits that let in-flight copies and MMAs finish before a CTA that is
// aborting releases its shared memory and tensor memory (independent of the wait limit).
constexpr uint64_t kDrainNs = 200ull * 1000 * 1000;

struct GblaSmem {
  float w[2][4 * 128];              // convolution taps (state: k, v; output: q)
  float gw[128];                    // output: half the norm weight
  float ss[4][128];                 // output: partial sums of squares of each row, per 32-column block
  uint64_t full[2][2];              // [ring][stage]: the stage's copies have landed
  uint64_t mma_done[2];             // per accumulator (the state kernel uses one)
  float red[kConsumerWarps];        // state: per-warp maximum gate logit of the chunk
  uint64_t wait_ns;                 // bound on every wait (the launch's wait limit)
  uint32_t tmem_slot;
  int abort;
};
constexpr size_t kStateSmem = 1024 + 5 * kPanel + 2 * kStateStage + sizeof(GblaSmem);
constexpr size_t kOutSmem = 1024 + 5 * kPanel + 2 * kQStage + 2 * kZStage + sizeof(GblaSmem);
static_assert(kStateSmem <= 227 * 1024 && kOutSmem <= 227 * 1024, "shared memory budget");

// Byte offset of 8-byte piece c4 (4 elements, c4 in 0..31) of row r of a 128-row bf16 tile held
// as two 64-column panels with the 128-byte swizzle (16-byte chunk index XOR row mod 8).
__device__ __forceinline__ uint32_t sw_off8(int r, int c4) {
  return (uint32_t)((c4 >> 4) * kPanel + r * 128 + ((((c4 >> 1) & 7) ^ (r & 7)) << 4) + ((c4 & 1) << 3));
}
// 16-byte chunk c (8 elements, c in 0..15) of row r of the same layout.
__device__ __forceinline__ uint32_t sw_off(int r, int c) {
  return (uint32_t)((c >> 3) * kPanel + r * 128 + (((c & 7) ^ (r & 7)) << 4));
}
// The same 8-byte piece of row r of a raw tile (two unswizzled 136-row panels).
__device__ __forceinline__ uint32_t raw_off8(int r, int c4) {
  return (uint32_t)((c4 >> 4) * kRawPanel + r * 128 + (c4 & 15) * 8);
}

// elu(x) + 1 = exp(min(x, 0)) + max(x, 0): no branch, one MUFU operation per element; two
// elements at a time on the packed fp32x2 path.
__device__ __forceinline__ void phi2(float& x0, float& x1) {
  float e0, e1;
  fmul2v(e0, e1, fminf(x0, 0.f), fminf(x1, 0.f), kLog2e, kLog2e);
  e0 = ex2(e0);
  e1 = ex2(e1);
  fadd2(e0, e1, fmaxf(x0, 0.f), fmaxf(x1, 0.f));
  x0 = e0, x1 = e1;
}
// w * (elu(x) + 1) = 2^(min(x, 0) log2 e + log2 w) + w max(x, 0), the gate w folded into the
// exponent (lw = log2 w; w = 0 gives lw = -inf and 0).
__device__ __forceinline__ void gated_phi2(float& x0, float& x1, float w, float lw) {
  float e0, e1;
  ffma2c(e0, e1, fminf(x0, 0.f), fminf(x1, 0.f), kLog2e, kLog2e, lw, lw);
  e0 = ex2(e0);
  e1 = ex2(e1);
  ffma2c(x0, x1, fmaxf(x0, 0.f), fmaxf(x1, 0.f), w, w, e0, e1);
}

__device__ __forceinline__ void unpack4(const uint2& u, float (&f)[4]) {
  const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
  const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
  f[0] = a.x, f[1] = a.y, f[2] = b.x, f[3] = b.y;
}
__device__ __forceinline__ void unpack8(const uint4& u, float (&f)[8]) {
  const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 t = __bfloat1622float2(b[i]);
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}
__device__ __forceinline__ uint2 pack4(const float (&v)[4]) {
  return make_uint2(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]));
}
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);   // .x (low half) = lo
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ uint2 pack4h(const float (&v)[4]) {
  return make_uint2(pack_f16x2(v[0], v[1]), pack_f16x2(v[2], v[3]));
}
__device__ __forceinline__ uint4 pack8(const float (&v)[8]) {
  uint4 u;
  u.x = pack_bf16x2(v[0], v[1]);
  u.y = pack_bf16x2(v[2], v[3]);
  u.z = pack_bf16x2(v[4], v[5]);
  u.w = pack_bf16x2(v[6], v[7]);
  return u;
}

__device__ __forceinline__ uint2 ld_shared_v2(uint32_t addr) {
  uint2 u;
  asm volatile("ld.shared.v2.b32 {%0, %1}, [%2];" : "=r"(u.x), "=r"(u.y) : "r"(addr));
  return u;
}
__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr) {
  uint4 u;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(u.x), "=r"(u.y), "=r"(u.z), "=r"(u.w) : "r"(addr));
  return u;
}
__device__ __forceinline__ void st_shared_v2(uint32_t addr, const uint2& u) {
  asm volatile("st.shared.v2.b32 [%0], {%1, %2};" ::"r"(addr), "r"(u.x), "r"(u.y) : "memory");
}

// One TMEM column of this warp's 32 lanes.
__device__ __forceinline__ float tmem_ld1(uint32_t taddr) {
  uint32_t r;
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];\n\ttcgen05.wait::ld.sync.aligned;"
               : "=r"(r)
               : "r"(taddr)
               : "memory");
  return __uint_as_float(r);
}

// Barrier of all 16 warps, returning whether `ok` holds in every thread.
__device__ __forceinline__ bool consumer_all(bool ok) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\tbar.red.and.pred q, 1, 512, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)ok)
      : "memory");
  return r != 0;
}
// Barrier of the four consumer warps that read TMEM lane quarter qd (warps qd, qd+4, qd+8, qd+12).
__device__ __forceinline__ void quarter_sync(int qd) { asm volatile("bar.sync %0, 128;" ::"r"(2 + qd) : "memory"); }

// Bounded wait on an mbarrier phase; false on timeout or when the CTA is aborting.  The first
// probe does not block; later probes suspend for at most 1 ms, and not at all under a limit
// below 100 us (a suspended probe may outlast a hint that short), so the limit is always seen.
__device__ __forceinline__ bool wait_phase(uint64_t* bar, uint32_t parity, GblaSmem& sm, uint32_t* status) {
  if (mbar_test(bar, parity)) return true;
  const uint64_t limit = sm.wait_ns;
  const bool spin = limit < 100000ull;
  const uint64_t t0 = global_ns();
  while (!(spin ? mbar_test(bar, parity) : mbar_test_suspend(bar, parity, 1000000u))) {
    if (*reinterpret_cast<volatile int*>(&sm.abort)) return false;
    if (global_ns() - t0 > limit) {
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
    if (global_ns() - t0 > kDrainNs) break;
}

// The causal convolution (width 4) of this thread's 8 rows (8g .. 8g+7 of the tile) and 4
// channels (piece c4) from a raw tile in shared memory whose row 8 is the tile's first token;
// tokens before the sequence start count as zero.  The 11 raw rows stream through once; output
// row i is handed to emit(i, x) as soon as its last tap has been added, so at most four rows of
// sums are live.
// `first` = the index of the first raw row at or after the sequence start (<= 0: all of them).
template <class Emit>
__device__ __forceinline__ void conv8(uint32_t raw, const float* taps, int c4, int g, int first, Emit&& emit) {
  float4 w[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) w[j] = *reinterpret_cast<const float4*>(taps + j * 128 + 4 * c4);
  float acc[kRowsT][4];
  const uint32_t src = raw + raw_off8(kRowsT * g + 5, c4);
#pragma unroll
  for (int m = 0; m < kRowsT + 3; ++m) {
    // Raw row m is token t0 + 8g - 3 + m; it meets tap j in output row i = m - 3 + j (the
    // output row's first contribution, tap 3, by a multiply).
    uint2 u = make_uint2(0u, 0u);
    if (m >= first) u = ld_shared_v2(src + m * 128);
    float f[4];
    unpack4(u, f);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int i = m - 3 + j;
      if (i >= 0 && i < kRowsT) {
        if (j == 3) {
          fmul2v(acc[i][0], acc[i][1], w[j].x, w[j].y, f[0], f[1]);
          fmul2v(acc[i][2], acc[i][3], w[j].z, w[j].w, f[2], f[3]);
        } else {
          ffma2v(acc[i][0], acc[i][1], w[j].x, w[j].y, f[0], f[1]);
          ffma2v(acc[i][2], acc[i][3], w[j].z, w[j].w, f[2], f[3]);
        }
      }
    }
    if (m >= 3) emit(m - 3, acc[m - 3]);
  }
}

__device__ __forceinline__ void tmem_alloc(uint32_t* slot, uint32_t cols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(slot)), "r"(cols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_free(uint32_t tmem, uint32_t cols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(cols) : "memory");
}

__device__ __forceinline__ void init_barriers(GblaSmem& sm, int nrings, uint64_t wait_ns) {
  for (int q = 0; q < nrings; ++q)
    for (int s = 0; s < 2; ++s) mbar_init(&sm.full[q][s], 1);   // thread 0's arrival + the copies' bytes
  mbar_init(&sm.mma_done[0], 1);
  mbar_init(&sm.mma_done[1], 1);
  sm.abort = 0;
  sm.wait_ns = wait_ns;
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// Row r of the third (64-column) panel of a 128-row operand tile: value x in its first column
// (fp16 or bf16), zeros elsewhere.
__device__ __forceinline__ void write_extra_row(uint8_t* panel, int r, float x, bool f16) {
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const uint32_t v0 = k == 0 ? (f16 ? pack_f16x2(x, 0.f) : pack_bf16x2(x, 0.f)) : 0u;
    st_shared_v4(smem_u32(panel) + r * 128 + ((k ^ (r & 7)) << 4), v0, 0u, 0u, 0u);
  }
}

// ---------------------------------------------------------------------------------------
// State: partial S and n of one chunk.  No producer warp: 16 warps (so up to 128 registers per
// thread); thread 0 issues the loads of tile i + 2 into the stage tile i used once the tile's
// barrier has shown every warp done with it.

__global__ void __launch_bounds__(kConsumers, 1) gbla_state_kernel(const __grid_constant__ GblaParams p) {
  extern __shared__ uint8_t dyn[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dyn) + 1023) & ~uintptr_t(1023));
  uint8_t* A = base;                // (w phi(k~)) tile: rows = tokens, columns = d (MN-major A)
  uint8_t* B = base + 2 * kPanel;   // [v~ | 1] tile: rows = tokens, columns = d + 16 (MN-major B)
  uint8_t* ring = base + 5 * kPanel;
  GblaSmem& sm = *reinterpret_cast<GblaSmem*>(ring + 2 * kStateStage);
  const GblaChunk ch = p.chunks[blockIdx.x];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = ch.head, lo = ch.seq_lo, hi = ch.seq_hi, H = p.H;
  if (tid == 0) init_barriers(sm, 1, p.wait_ns);
  for (int i = tid; i < 4 * 128; i += kConsumers) {
    sm.w[0][i] = p.conv_k[h * 4 * 128 + i];
    sm.w[1][i] = p.conv_v[h * 4 * 128 + i];
  }
  // The ones column: n = sum over tokens of w phi(k~) comes out of the MMA as column d.
  if (tid < 128) write_extra_row(B + 2 * kPanel, tid, 1.f, true);
  if (warp == 0) tmem_alloc(&sm.tmem_slot, 256);
  const __nv_bfloat16* ax = reinterpret_cast<const __nv_bfloat16*>(p.a);
  {
    // The chunk's largest gate logit (for the operand scale below).
    const int t_lo = lo + ch.tile0 * 128, t_hi = min(hi, lo + (ch.tile0 + ch.n_tiles) * 128);
    float amax = -INFINITY;
    for (int t = t_lo + tid; t < t_hi; t += kConsumers) amax = fmaxf(amax, __bfloat162float(ax[(int64_t)t * H + h]));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    if (lane == 0) sm.red[warp] = amax;
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_slot;
  // Operand scale 2^es: the chunk's largest gate w_max = sigmoid(max a) times 2^es lies in
  // (1/2, 1], so w phi(k~) keeps fp16's range whatever the gates (a chunk of nearly closed gates
  // would otherwise underflow to 0); the partial state and n are divided by 2^es (exactly) at
  // the end.  es = floor(-log2 w_max) = floor(log2(1 + 2^(-max a log2 e))), at most 100.
  int es;
  {
    float amax = sm.red[0];
#pragma unroll
    for (int w = 1; w < kConsumerWarps; ++w) amax = fmaxf(amax, sm.red[w]);
    const float l = lg2_approx(1.f + ex2(-amax * kLog2e));
    es = l < 100.f ? (int)l : 100;
  }
  // Tile t's k and v (two panels each, from 8 rows before the tile) into stage t % 2.
  auto issue = [&](int t) {
    const int s = t & 1, y0 = ch.seq_lo + (ch.tile0 + t) * 128;
    uint8_t* st = ring + s * kStateStage;
    mbar_expect_tx(&sm.full[0][s], kStateStage);
#pragma unroll
    for (int pn = 0; pn < 2; ++pn) {
      tma_load_2d(st + pn * kRawPanel, &p.tm_k, h * 128 + pn * 64, y0 - 8, &sm.full[0][s]);
      tma_load_2d(st + (2 + pn) * kRawPanel, &p.tm_v, h * 128 + pn * 64, y0 - 8, &sm.full[0][s]);
    }
  };
  int issued = 0;
  if (tid == 0) {
    prefetch_tmap(&p.tm_k);
    prefetch_tmap(&p.tm_v);
    for (; issued < 2 && issued < ch.n_tiles; ++issued) issue(issued);
  }
  const int g = warp, c4 = lane;
  // fp16 operands (A and B of one type, as kind::f16 requires): the rounding of w phi(k~) and
  // v~ is the largest error of the layer (the output's RMS normalisation magnifies it in rows
  // whose weighted average nearly cancels), and fp16 has 3 more mantissa bits than bf16; both
  // stay far inside its range (|w phi(k~)|, |v~| < 65504).
  constexpr uint32_t idesc = make_idesc(128, kN, true, true) & ~((7u << 7) | (7u << 10));
  bool ok = true;
  int done = 0;
  // The gate of row r of this warp's rows is computed by lanes r, r + 8, ... (its logit loaded
  // one tile ahead; -inf past the sequence end, giving w = 0) and read by shuffles.
  const int gl = lane & 7;
  auto load_gate = [&](int tile) -> float {
    const int tok = lo + (ch.tile0 + tile) * 128 + kRowsT * g + gl;
    return (tile < ch.n_tiles && tok < hi) ? __bfloat162float(ax[(int64_t)tok * H + h]) : -INFINITY;
  };
  float a_next = load_gate(0);
  for (int i = 0; i < ch.n_tiles; ++i) {
    const int s = i & 1;
    const uint32_t raw = smem_u32(ring + s * kStateStage);
    // Raw rows before `first` precede the sequence start (only in its first tile).
    const int first = 3 - kRowsT * g - 128 * (ch.tile0 + i);
    const float a = a_next;
    a_next = load_gate(i + 1);
    // log2 w = -log2(1 + 2^(-a log2 e)) for w = sigmoid(a), and the scaled gate 2^(log2 w + es)
    // (exact in relative terms however small w is); row r's pair is read from lane r.
    const float lw_l = (float)es - lg2_approx(1.f + ex2(-a * kLog2e)), w_l = ex2(lw_l);
    ok = wait_phase(&sm.full[0][s], (i >> 1) & 1, sm, p.status);
    uint2 uk[kRowsT], uv[kRowsT];
    // Both operand tiles into registers first (no wait between the two convolutions, so they
    // can interleave), then stored once the previous tile's MMAs have read the buffers.
    conv8(raw, sm.w[0], c4, g, first, [&](int r, float (&x)[4]) {
      const float wr = __shfl_sync(0xffffffffu, w_l, r), lwr = __shfl_sync(0xffffffffu, lw_l, r);
      gated_phi2(x[0], x[1], wr, lwr);
      gated_phi2(x[2], x[3], wr, lwr);
      uk[r] = pack4h(x);
    });
    conv8(raw + 2 * kRawPanel, sm.w[1], c4, g, first, [&](int r, float (&x)[4]) { uv[r] = pack4h(x); });
    if (ok && i > 0) ok = wait_phase(&sm.mma_done[0], (i - 1) & 1, sm, p.status);
    if (ok) {
#pragma unroll
      for (int r = 0; r < kRowsT; ++r) {
        st_shared_v2(smem_u32(A) + sw_off8(kRowsT * g + r, c4), uk[r]);
        st_shared_v2(smem_u32(B) + sw_off8(kRowsT * g + r, c4), uv[r]);
      }
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    // One barrier per tile: the operands are complete, every thread's waits succeeded, and no
    // warp reads stage s any more.
    if (!consumer_all(ok)) {
      ok = false;
      break;
    }
    if (warp == 0) {
      if (lane == 0 && i + 2 < ch.n_tiles) {
        issue(i + 2);
        ++issued;
      }
      tc_fence_after();
      const uint64_t ad = sdesc_sw128(smem_u32(A), kPanel, 1024), bd = sdesc_sw128(smem_u32(B), kPanel, 1024);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        mma_ss_w(tmem, ad + (uint64_t)(kk * 2048 / 16), bd + (uint64_t)(kk * 2048 / 16), idesc,
                 (i > 0 || kk > 0) ? 1u : 0u);
      tc_commit_w(&sm.mma_done[0]);
    }
    done = i + 1;
  }
  if (tid == 0 && !ok) {
    // Aborting: let the loads in flight land before the CTA releases its shared memory.
    for (int t = (issued > 2 ? issued - 2 : 0); t < issued; ++t) drain_phase(&sm.full[0][t & 1], (t >> 1) & 1);
  }
  if (done > 0) {
    if (ok) ok = wait_phase(&sm.mma_done[0], (done - 1) & 1, sm, p.status);
    else drain_phase(&sm.mma_done[0], (done - 1) & 1);
  }
  ok = consumer_all(ok);
  tc_fence_after();
  float* part = p.part_s + (int64_t)blockIdx.x * (128 * 128 + 128);
  {
    // Row i = 32 * (warp % 4) + lane of the partial state (channel i of phi(k~)), columns
    // 32 * (warp / 4) .. +31 (v channels): one 32-column TMEM load per warp; column d is n.
    const int qd = warp & 3, cb = warp >> 2;
    const int i = 32 * qd + lane;
    const bool keep = ok && done > 0;
    const float unscale = __int_as_float((127 - es) << 23);   // 2^-es
    float4* dst = reinterpret_cast<float4*>(part + (int64_t)i * 128 + 32 * cb);
    uint32_t r[32];
    tmem_ld32(tmem + ((uint32_t)(32 * qd) << 16) + 32 * cb, r);
#pragma unroll
    for (int e = 0; e < 8; ++e)
      dst[e] = keep ? make_float4(__uint_as_float(r[4 * e]) * unscale, __uint_as_float(r[4 * e + 1]) * unscale,
                                  __uint_as_float(r[4 * e + 2]) * unscale, __uint_as_float(r[4 * e + 3]) * unscale)
                    : make_float4(0.f, 0.f, 0.f, 0.f);
    if (cb == 0) {
      const float nv = tmem_ld1(tmem + ((uint32_t)(32 * qd) << 16) + 128);
      part[128 * 128 + i] = keep ? nv * unscale : 0.f;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_free(tmem, 256);
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
// Output: y for every token of one chunk.  The MMA of tile i runs while the epilogue of tile
// i - 1 reads the other TMEM accumulator; q and z come through separate rings because z is
// needed one tile later than q.

__global__ void __launch_bounds__(kConsumers, 1) gbla_out_kernel(const __grid_constant__ GblaParams p) {
  extern __shared__ uint8_t dyn[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dyn) + 1023) & ~uintptr_t(1023));
  uint8_t* A = base;                 // phi(q~) tile: rows = tokens, columns = d (K-major A)
  uint8_t* Bs = base + 2 * kPanel;   // [S | n]: rows = phi channels (K), columns = v channels + n (MN-major B)
  uint8_t* qring = base + 5 * kPanel;
  uint8_t* zring = qring + 2 * kQStage;
  GblaSmem& sm = *reinterpret_cast<GblaSmem*>(zring + 2 * kZStage);
  const GblaChunk ch = p.chunks[blockIdx.x];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = ch.head, lo = ch.seq_lo, hi = ch.seq_hi, H = p.H;
  if (tid == 0) init_barriers(sm, 2, p.wait_ns);
  if (warp == 0) tmem_alloc(&sm.tmem_slot, 512);
  {
    // S of this (sequence, head) into the B tile: rows 8w .. 8w+7, 8-byte piece `lane`.
    const uint2* src = reinterpret_cast<const uint2*>(p.state + (int64_t)ch.pair * 128 * 128);
#pragma unroll
    for (int r = 0; r < kRowsT; ++r) {
      const int row = kRowsT * warp + r;
      st_shared_v2(smem_u32(Bs) + sw_off8(row, lane), src[row * 32 + lane]);
    }
  }
  // n as the first column of the third panel: the MMA's column d is n . phi(q~).
  if (tid < 128) write_extra_row(Bs + 2 * kPanel, tid, p.norm_n[(int64_t)ch.pair * 128 + tid], false);
  for (int i = tid; i < 4 * 128; i += kConsumers) sm.w[0][i] = p.conv_q[h * 4 * 128 + i];
  if (tid < 128) sm.gw[tid] = 0.5f * p.norm_w[h * 128 + tid];   // g / 2 (see the epilogue)
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_slot;
  // No producer warp: thread 0 issues the copies.  q of tile t goes into q stage t % 2 once
  // every warp has convolved tile t - 2 (the tile barrier of iteration t - 2); z of tile t into
  // z stage t % 2 once the epilogue of tile t - 2 is done (the tile barrier of iteration t).
  auto issue_q = [&](int t) {
    const int s = t & 1, y0 = ch.seq_lo + (ch.tile0 + t) * 128;
    mbar_expect_tx(&sm.full[0][s], kQStage);
#pragma unroll
    for (int pn = 0; pn < 2; ++pn)
      tma_load_2d(qring + s * kQStage + pn * kRawPanel, &p.tm_q, h * 128 + pn * 64, y0 - 8, &sm.full[0][s]);
  };
  auto issue_z = [&](int t) {
    const int s = t & 1, y0 = ch.seq_lo + (ch.tile0 + t) * 128;
    mbar_expect_tx(&sm.full[1][s], kZStage);
#pragma unroll
    for (int pn = 0; pn < 2; ++pn)
      tma_load_2d(zring + s * kZStage + pn * kPanel, &p.tm_z, h * 128 + pn * 64, y0, &sm.full[1][s]);
  };
  int q_issued = 0, z_issued = 0;
  if (tid == 0) {
    prefetch_tmap(&p.tm_q);
    prefetch_tmap(&p.tm_z);
    prefetch_tmap(&p.tm_y);
    for (; q_issued < 2 && q_issued < ch.n_tiles; ++q_issued) issue_q(q_issued);
    for (; z_issued < 2 && z_issued < ch.n_tiles; ++z_issued) issue_z(z_issued);
  }
  {
    const int g = warp, c4 = lane;
    __nv_bfloat16* yx = reinterpret_cast<__nv_bfloat16*>(p.y);
    constexpr uint32_t idesc = make_idesc(128, kN, true);
    // Epilogue roles: warp w reads the TMEM rows of its lane quarter qd = w % 4 (rows 32 qd ..
    // 32 qd + 31) and the 32 columns of block cb = w / 4.
    const int qd = warp & 3, cb = warp >> 2;
    const int r = 32 * qd + lane;
    bool ok = true, stores_pending = false;
    int done = 0;

    // Epilogue of tile j: y = o / den / rms * g * silu(z), written over z in its stage (row
    // quarters that lie entirely inside the sequence, then bulk tensor stores) or straight to
    // y with 16-byte stores (a quarter that reaches past the sequence end).
    auto epilogue = [&](int j) {
      const int zs = j & 1;
      const int64_t t0 = (int64_t)lo + (int64_t)(ch.tile0 + j) * 128;
      const bool zok = wait_phase(&sm.full[1][zs], (j >> 1) & 1, sm, p.status);
      tc_fence_after();
      const uint32_t acc = tmem + (uint32_t)(j & 1) * kAccStride + ((uint32_t)(32 * qd) << 16);
      const int64_t t = t0 + r;
      const bool live = zok && t < hi;
      const bool whole = zok && t0 + 32 * qd + 31 < hi;
      uint32_t v[32];
      tmem_ld32(acc + 32 * cb, v);
      const float inv_den = 1.f / (tmem_ld1(acc + 128) + kEpsAttn);
      tc_fence_before();
      float s0 = 0.f, s1 = 0.f;
#pragma unroll
      for (int e = 0; e < 32; e += 2)
        ffma2v(s0, s1, __uint_as_float(v[e]), __uint_as_float(v[e + 1]), __uint_as_float(v[e]), __uint_as_float(v[e + 1]));
      sm.ss[cb][r] = (s0 + s1) * inv_den * inv_den;
      quarter_sync(qd);
      const float ss = sm.ss[0][r] + sm.ss[1][r] + sm.ss[2][r] + sm.ss[3][r];
      const float scale = inv_den * rsqrtf(ss * (1.f / 128.f) + kEpsNorm);
      const uint32_t zt = smem_u32(zring + zs * kZStage);
      uint4* yrow = reinterpret_cast<uint4*>(yx + (live ? (t * H + h) * 128 : 0));
#pragma unroll
      for (int k4 = 0; k4 < 4; ++k4) {
        const int chunk = 4 * cb + k4;   // 16-byte chunk (8 columns) of the row
        const uint32_t za = zt + sw_off(r, chunk);
        float zf[8], yv[8];
        unpack8(ld_shared_v4(za), zf);
        const float4 g0 = *reinterpret_cast<const float4*>(sm.gw + 8 * chunk);
        const float4 g1 = *reinterpret_cast<const float4*>(sm.gw + 8 * chunk + 4);
        const float gg[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
#pragma unroll
        for (int e = 0; e < 8; e += 2) {
          // y = o * scale * g * silu(z) with g * silu(z) = u + u tanh(z / 2), u = z g / 2 (the
          // shared memory holds g / 2), on packed pairs.
          float u0, u1, h0, h1, o0, o1;
          fmul2v(u0, u1, zf[e], zf[e + 1], gg[e], gg[e + 1]);
          fmul2v(h0, h1, zf[e], zf[e + 1], 0.5f, 0.5f);
          h0 = tanh_approx(h0);
          h1 = tanh_approx(h1);
          ffma2c(h0, h1, h0, h1, u0, u1, u0, u1);
          fmul2v(o0, o1, __uint_as_float(v[8 * k4 + e]), __uint_as_float(v[8 * k4 + e + 1]), scale, scale);
          fmul2v(yv[e], yv[e + 1], h0, h1, o0, o1);
        }
        const uint4 yu = pack8(yv);
        if (whole) st_shared_v4(za, yu.x, yu.y, yu.z, yu.w);
        else if (live) yrow[chunk] = yu;
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      quarter_sync(qd);
      // Warps of column blocks 0 and 2, lane 0: one bulk tensor store of this quarter's rows per
      // 64-column panel; the stage is released once the stores have read it.
      if ((cb & 1) == 0 && lane == 0 && whole) {
        const int pn = cb >> 1;
        tma_store_2d(&p.tm_y, zring + zs * kZStage + pn * kPanel + 32 * qd * 128, h * 128 + pn * 64, (int)(t0 + 32 * qd));
        bulk_commit();
        bulk_wait_read();
        stores_pending = true;
      }
      __syncwarp();
    };

    for (int i = 0; i < ch.n_tiles; ++i) {
      const int s = i & 1;
      const bool landed = wait_phase(&sm.full[0][s], (i >> 1) & 1, sm, p.status);
      ok = landed;
      uint2 uq[kRowsT];
      conv8(smem_u32(qring + s * kQStage), sm.w[0], c4, g, 3 - kRowsT * g - 128 * (ch.tile0 + i),
            [&](int rr, float (&x)[4]) {
              phi2(x[0], x[1]);
              phi2(x[2], x[3]);
              uq[rr] = pack4(x);
            });
      // The previous tile's MMAs must have read A (and finished its accumulator) first.
      if (ok && i > 0) ok = wait_phase(&sm.mma_done[(i - 1) & 1], ((i - 1) >> 1) & 1, sm, p.status);
      if (ok) {
#pragma unroll
        for (int rr = 0; rr < kRowsT; ++rr) st_shared_v2(smem_u32(A) + sw_off8(kRowsT * g + rr, c4), uq[rr]);
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      // One barrier per tile: A is complete, and every thread's waits succeeded.
      if (!consumer_all(ok)) {
        ok = false;
        break;
      }
      if (warp == 0) {
        if (lane == 0) {
          if (i + 2 < ch.n_tiles) {
            issue_q(i + 2);
            ++q_issued;
          }
          if (i >= 2) {
            issue_z(i);
            ++z_issued;
          }
        }
        tc_fence_after();
        const uint64_t ad = sdesc_sw128(smem_u32(A), 16, 1024), bd = sdesc_sw128(smem_u32(Bs), kPanel, 1024);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {   // 16 channels per step
          const uint64_t aoff = (uint64_t)(((kk >> 2) * kPanel + (kk & 3) * 32) >> 4);
          mma_ss_w(tmem + (uint32_t)s * kAccStride, ad + aoff, bd + (uint64_t)(kk * 2048 / 16), idesc, kk > 0 ? 1u : 0u);
        }
        tc_commit_w(&sm.mma_done[s]);
      }
      if (i > 0) epilogue(i - 1);
      done = i + 1;
    }
    if (tid == 0 && !ok) {
      // Aborting: let the copies in flight land before the CTA releases its shared memory.
      for (int t = (q_issued > 2 ? q_issued - 2 : 0); t < q_issued; ++t) drain_phase(&sm.full[0][t & 1], (t >> 1) & 1);
      for (int t = (z_issued > 2 ? z_issued - 2 : 0); t < z_issued; ++t) drain_phase(&sm.full[1][t & 1], (t >> 1) & 1);
    }
    if (done > 0) {
      const int j = done - 1;
      if (ok) ok = wait_phase(&sm.mma_done[j & 1], (j >> 1) & 1, sm, p.status);
      else drain_phase(&sm.mma_done[j & 1], (j >> 1) & 1);
      if (consumer_all(ok)) epilogue(j);
    }
    if (stores_pending) bulk_wait_all();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_free(tmem, 512);
}

}  // namespace

cudaError_t launch_gbla(const GblaParams& p, int n_chunks, int n_pairs, cudaStream_t s) {
  if (n_chunks <= 0) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(gbla_state_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kStateSmem);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(gbla_out_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kOutSmem);
  if (e != cudaSuccess) return e;
  gbla_state_kernel<<<n_chunks, kConsumers, kStateSmem, s>>>(p);
  gbla_reduce_kernel<<<dim3(n_pairs, (128 * 128 + 128 + 255) / 256), 256, 0, s>>>(p);
  gbla_out_kernel<<<n_chunks, kConsumers, kOutSmem, s>>>(p);
  return cudaGetLastError();
}

}  // namespace bat
