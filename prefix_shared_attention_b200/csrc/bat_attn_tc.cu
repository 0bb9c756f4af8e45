// Bipartite prefix-shared attention forward on tcgen05 tensor cores (sm_100a).
//
// Operation (Bat lead page, sections "This paper's idea" and "Why it works"): each
// request's suffix rows attend, with no mask, over [cached prefix K/V ; own suffix K/V].
// The prefix K/V is computed once and cached; every request that references it reuses it.
//
// One persistent CTA per SM walks the work list built by the host grouping pass.  A work
// item holds one head and up to two 128-row query tiles (A, B) that read the same prefix.
// The CTA streams the item's key tiles through shared memory with TMA, once each, and both
// query tiles consume every shared tile:
//
//   warp 8       TMA producer: Q tiles, then K/V tiles in stream order into a ring
//   warp 9       MMA issuer (one lane): S = Q.K^T (SS) and O += P.V (TS, P read from TMEM)
//   warps 0..3   softmax + epilogue of tile A (one thread per query row = TMEM lane)
//   warps 4..7   softmax + epilogue of tile B
//
// TMEM (512 columns): S_A, S_B (128 fp32 columns each), O_A, O_B (d columns each); P (bf16
// pairs, 64 columns) aliases S when d = 128, and has its own columns when d = 64.
// The softmax is online in the base-2 domain with a lazily updated reference maximum: the
// accumulator is rescaled only when a row's maximum grows by more than kRescaleThreshold,
// which is exact because O and the row sum l always share the same reference.
//
// Every spin-wait is bounded (wall clock); on expiry the CTA raises a CTA-wide abort flag,
// records the failure in the device status word, drains its in-flight copies and MMAs,
// frees its TMEM and returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "bat_kernels.h"

namespace bat {
namespace {

__device__ uint32_t g_status_word;

constexpr float kRescaleThreshold = 8.0f;   // log2 units: P stays <= 2^8 between rescales
constexpr uint64_t kDrainNs = 200ull * 1000 * 1000;

// ------------------------------------------------------------------------------------
// PTX wrappers

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(
                   smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// D[tmem] (+)= A[smem desc] * B[smem desc]
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem desc]
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 32 consecutive fp32 columns of this thread's TMEM lane, waited for in the same statement
// so no use of the registers can be scheduled before the data has arrived.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}

__device__ __forceinline__ void tmem_ld128(uint32_t taddr, uint32_t (&r)[128]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x128.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, %48, %49, %50, %51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, %62, %63, %64, %65, %66, %67, %68, %69, %70, %71, %72, %73, %74, %75, %76, %77, %78, %79, %80, %81, %82, %83, %84, %85, %86, %87, %88, %89, %90, %91, %92, %93, %94, %95, %96, %97, %98, %99, %100, %101, %102, %103, %104, %105, %106, %107, %108, %109, %110, %111, %112, %113, %114, %115, %116, %117, %118, %119, %120, %121, %122, %123, %124, %125, %126, %127}, [%128];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]), "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]), "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63]), "=r"(r[64]), "=r"(r[65]), "=r"(r[66]), "=r"(r[67]), "=r"(r[68]), "=r"(r[69]), "=r"(r[70]), "=r"(r[71]), "=r"(r[72]), "=r"(r[73]), "=r"(r[74]), "=r"(r[75]), "=r"(r[76]), "=r"(r[77]), "=r"(r[78]), "=r"(r[79]), "=r"(r[80]), "=r"(r[81]), "=r"(r[82]), "=r"(r[83]), "=r"(r[84]), "=r"(r[85]), "=r"(r[86]), "=r"(r[87]), "=r"(r[88]), "=r"(r[89]), "=r"(r[90]), "=r"(r[91]), "=r"(r[92]), "=r"(r[93]), "=r"(r[94]), "=r"(r[95]), "=r"(r[96]), "=r"(r[97]), "=r"(r[98]), "=r"(r[99]), "=r"(r[100]), "=r"(r[101]), "=r"(r[102]), "=r"(r[103]), "=r"(r[104]), "=r"(r[105]), "=r"(r[106]), "=r"(r[107]), "=r"(r[108]), "=r"(r[109]), "=r"(r[110]), "=r"(r[111]), "=r"(r[112]), "=r"(r[113]), "=r"(r[114]), "=r"(r[115]), "=r"(r[116]), "=r"(r[117]), "=r"(r[118]), "=r"(r[119]), "=r"(r[120]), "=r"(r[121]), "=r"(r[122]), "=r"(r[123]), "=r"(r[124]), "=r"(r[125]), "=r"(r[126]), "=r"(r[127])
      : "r"(taddr)
      : "memory");
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};"
      :
      : "r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);   // .x (low half) = lo
  return *reinterpret_cast<uint32_t*>(&v);
}

// Shared-memory matrix descriptor, 128-byte swizzle (tcgen05 format: version 1 at bit 46,
// layout type 2 = SWIZZLE_128B at bits 61..63).
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

// Instruction descriptor, kind::f16: D f32, A and B bf16, A K-major, B K- or MN-major.
__host__ __device__ constexpr uint32_t make_idesc(int M, int N, bool b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((b_mn_major ? 1u : 0u) << 16) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}

// ------------------------------------------------------------------------------------
// Compile-time layout

template <int D>
struct Cfg {
  static constexpr int kPanels = D / 64;                 // 64-element (128-byte) column panels
  static constexpr int kPanelBytes = kTileM * 128;       // 128 rows x 128 bytes
  static constexpr int kTileBytes = kPanels * kPanelBytes;
  static constexpr int kStages = D == 128 ? 4 : 8;        // K/V ring depth
  static constexpr bool kAliasP = D == 128;               // P overwrites S in TMEM
  static constexpr uint32_t kTmemCols = 512;
  __host__ __device__ static constexpr uint32_t s_col(int x) { return 128u * x; }
  __host__ __device__ static constexpr uint32_t o_col(int x) { return 256u + (uint32_t)D * x; }
  __host__ __device__ static constexpr uint32_t p_col(int x) { return kAliasP ? 128u * x : 384u + 64u * x; }
  static constexpr uint32_t kIdescS = make_idesc(128, 128, false);
  static constexpr uint32_t kIdescPV = make_idesc(128, D, true);
  static constexpr int kBarBytes = 8 * (2 * kStages + 2 * 6 + 1) + 16;
  static constexpr size_t kSmemBytes = 1024 + (size_t)(2 + kStages) * kTileBytes + kBarBytes;
};

// The key tiles an item streams: prefix tiles (read by every query tile of the item), then
// suffix tiles (shared when both query tiles belong to one request, else interleaved A, B).
struct Stream {
  int npre, nsA, nsB, n, nq;
  bool shared;
  __device__ __forceinline__ explicit Stream(const WorkItem& w) {
    npre = (w.pre_len + kTileN - 1) / kTileN;
    nq = w.n_q;
    shared = w.shared != 0 || w.n_q == 1;
    nsA = (w.sA_len + kTileN - 1) / kTileN;
    nsB = shared ? 0 : (w.sB_len + kTileN - 1) / kTileN;
    n = npre + nsA + nsB;
  }
  __device__ __forceinline__ int count(int x) const { return npre + (shared || x == 0 ? nsA : nsB); }
  // Global tile j: consumer mask (bit x = query tile x), source, first row.
  __device__ __forceinline__ void tile(const WorkItem& w, int j, int& mask, bool& from_cache, int& row0) const {
    if (j < npre) {
      mask = nq == 2 ? 3 : 1;
      from_cache = true;
      row0 = w.pre_row0 + j * kTileN;
      return;
    }
    const int k = j - npre;
    from_cache = false;
    if (shared) {
      mask = nq == 2 ? 3 : 1;
      row0 = w.sA_row0 + k * kTileN;
      return;
    }
    const int mm = nsA < nsB ? nsA : nsB;
    int x, idx;
    if (k < 2 * mm) {
      x = k & 1;
      idx = k >> 1;
    } else {
      x = nsA > nsB ? 0 : 1;
      idx = mm + (k - 2 * mm);
    }
    mask = 1 << x;
    row0 = (x ? w.sB_row0 : w.sA_row0) + idx * kTileN;
  }
  // Valid keys in the t-th tile that query tile x consumes.
  __device__ __forceinline__ int valid(const WorkItem& w, int x, int t) const {
    if (t < npre) return min(kTileN, w.pre_len - t * kTileN);
    const int len = (shared || x == 0) ? w.sA_len : w.sB_len;
    return min(kTileN, len - (t - npre) * kTileN);
  }
};

struct Ctl {
  volatile int* abort_flag;
  uint32_t* status;
  uint64_t limit_ns;
};

// Bounded wait on an mbarrier phase, uniform across the warp (every lane calls it).
// Returns false when the CTA is aborting (this wait timed out, or another one did).
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, const Ctl& c) {
  bool ok = mbar_test(bar, parity);
  if (!ok) {
    const uint64_t t0 = global_ns();
    while (true) {
#pragma unroll 1
      for (int i = 0; i < 16 && !ok; ++i) ok = mbar_test(bar, parity);
      if (ok) break;
      if (*c.abort_flag) break;
      if (global_ns() - t0 > c.limit_ns) {
        *c.abort_flag = 1;
        atomicOr(c.status, 1u);
        break;
      }
    }
  }
  return __all_sync(0xffffffffu, ok);
}

// Bounded wait used while draining after an abort (ignores the abort flag).
__device__ __forceinline__ void drain_bar(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = global_ns();
  while (!mbar_test(bar, parity)) {
    if (global_ns() - t0 > kDrainNs) break;
  }
}

template <int D>
struct Smem {
  uint8_t* q;        // [2][kTileBytes]
  uint8_t* kv;       // [kStages][kTileBytes]
  uint64_t* kv_full;
  uint64_t* kv_empty;
  uint64_t* q_full;   // [2]
  uint64_t* q_empty;  // [2]
  uint64_t* s_full;   // [2]
  uint64_t* s_free;   // [2]
  uint64_t* p_full;   // [2]
  uint64_t* pv_done;  // [2]
  uint64_t* drain;
  uint32_t* tmem_slot;
  volatile int* abort_flag;
};

// ------------------------------------------------------------------------------------
// Roles

template <int D>
__device__ void producer_role(const TcParams& p, const Smem<D>& sm, const Ctl& ctl) {
  using C = Cfg<D>;
  const int lane = threadIdx.x & 31;
  uint32_t ring = 0, qcnt[2] = {0, 0};
  bool ok = true;
  for (int64_t it = blockIdx.x; ok && it < p.n_items; it += gridDim.x) {
    const WorkItem w = p.items[it];
    for (int x = 0; ok && x < w.n_q; ++x) {
      ok = wait_bar(sm.q_empty + x, (qcnt[x] & 1) ^ 1, ctl);
      if (!ok) break;
      if (lane == 0) {
        mbar_expect_tx(sm.q_full + x, C::kTileBytes);
        const int row0 = x ? w.qB_row0 : w.qA_row0;
#pragma unroll
        for (int pn = 0; pn < C::kPanels; ++pn)
          tma_load_2d(sm.q + x * C::kTileBytes + pn * C::kPanelBytes, &p.tm_q, w.head * D + pn * 64, row0,
                      sm.q_full + x);
      }
      __syncwarp();
      ++qcnt[x];
    }
    const Stream st(w);
    for (int j = 0; ok && j < st.n; ++j) {
      int mask, row0;
      bool from_cache;
      st.tile(w, j, mask, from_cache, row0);
      for (int kv = 0; kv < 2; ++kv) {
        const uint32_t s = ring % C::kStages, ph = (ring / C::kStages) & 1;
        ok = wait_bar(sm.kv_empty + s, ph ^ 1, ctl);
        if (!ok) break;
        if (lane == 0) {
          const CUtensorMap* m = from_cache ? (kv ? &p.tm_vc : &p.tm_kc) : (kv ? &p.tm_vs : &p.tm_ks);
          mbar_expect_tx(sm.kv_full + s, C::kTileBytes);
#pragma unroll
          for (int pn = 0; pn < C::kPanels; ++pn)
            tma_load_2d(sm.kv + s * C::kTileBytes + pn * C::kPanelBytes, m, w.head * D + pn * 64, row0,
                        sm.kv_full + s);
        }
        __syncwarp();
        ++ring;
      }
    }
  }
  if (!ok && lane == 0) {
    // Let every copy this warp issued land before the CTA releases its shared memory.
    const uint32_t n = ring < (uint32_t)C::kStages ? ring : (uint32_t)C::kStages;
    for (uint32_t i = ring - n; i < ring; ++i) drain_bar(sm.kv_full + i % C::kStages, (i / C::kStages) & 1);
    for (int x = 0; x < 2; ++x)
      if (qcnt[x]) drain_bar(sm.q_full + x, (qcnt[x] - 1) & 1);
  }
  __syncwarp();
}

template <int D>
__device__ void mma_role(const TcParams& p, const Smem<D>& sm, const Ctl& ctl, uint32_t tmem) {
  using C = Cfg<D>;
  const int lane = threadIdx.x & 31;
  uint32_t ring = 0, qcnt[2] = {0, 0}, s_issued[2] = {0, 0}, pv_issued[2] = {0, 0}, p_seen[2] = {0, 0};
  bool ok = true;
  const uint32_t q_base = smem_u32(sm.q), kv_base = smem_u32(sm.kv);
  for (int64_t it = blockIdx.x; ok && it < p.n_items; it += gridDim.x) {
    const WorkItem w = p.items[it];
    const Stream st(w);
    int s_left[2] = {st.count(0), w.n_q == 2 ? st.count(1) : 0};
    bool first_s[2] = {true, true}, first_pv[2] = {true, true};
    const uint32_t ring0 = ring;

    auto do_s = [&](int j) {
      int mask, row0;
      bool from_cache;
      st.tile(w, j, mask, from_cache, row0);
      const uint32_t rk = ring0 + 2u * j, s = rk % C::kStages;
      ok = wait_bar(sm.kv_full + s, (rk / C::kStages) & 1, ctl);
      if (!ok) return;
      for (int x = 0; x < 2; ++x) {
        if (!((mask >> x) & 1)) continue;
        if (first_s[x]) {
          ok = wait_bar(sm.q_full + x, qcnt[x] & 1, ctl);
          if (!ok) return;
          ++qcnt[x];
          first_s[x] = false;
        }
        if (s_issued[x] > 0) {
          // The S columns are free once the previous P (aliased) was consumed, or once the
          // softmax finished reading the previous S (separate P columns).
          if (C::kAliasP) ok = wait_bar(sm.pv_done + x, (pv_issued[x] - 1) & 1, ctl);
          else ok = wait_bar(sm.s_free + x, (s_issued[x] - 1) & 1, ctl);
          if (!ok) return;
        }
        tc_fence_after();
        if (lane == 0) {
          const uint32_t qa = q_base + x * C::kTileBytes, kb = kv_base + s * C::kTileBytes;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * C::kPanelBytes + (kk & 3) * 32;
            mma_ss(tmem + C::s_col(x), sdesc_sw128(qa + off, 16, 1024), sdesc_sw128(kb + off, 16, 1024),
                   C::kIdescS, kk > 0 ? 1u : 0u);
          }
          tc_commit(sm.s_full + x);
          if (s_left[x] == 1) tc_commit(sm.q_empty + x);
        }
        __syncwarp();
        --s_left[x];
        ++s_issued[x];
      }
      if (lane == 0) tc_commit(sm.kv_empty + s);
      __syncwarp();
    };

    auto do_pv = [&](int j) {
      int mask, row0;
      bool from_cache;
      st.tile(w, j, mask, from_cache, row0);
      const uint32_t rv = ring0 + 2u * j + 1, s = rv % C::kStages;
      ok = wait_bar(sm.kv_full + s, (rv / C::kStages) & 1, ctl);
      if (!ok) return;
      for (int x = 0; x < 2; ++x) {
        if (!((mask >> x) & 1)) continue;
        ok = wait_bar(sm.p_full + x, p_seen[x] & 1, ctl);
        if (!ok) return;
        ++p_seen[x];
        tc_fence_after();
        if (lane == 0) {
          const uint32_t vb = kv_base + s * C::kTileBytes;
#pragma unroll
          for (int kk = 0; kk < kTileN / 16; ++kk) {
            // V tile is MN-major for this product: 16 keys = two 8-row swizzle groups (2 KiB);
            // LBO steps between 64-column panels, SBO between 8-row groups.
            mma_ts(tmem + C::o_col(x), tmem + C::p_col(x) + kk * 8, sdesc_sw128(vb + kk * 2048, C::kPanelBytes, 1024),
                   C::kIdescPV, (first_pv[x] && kk == 0) ? 0u : 1u);
          }
          tc_commit(sm.pv_done + x);
        }
        __syncwarp();
        first_pv[x] = false;
        ++pv_issued[x];
      }
      if (lane == 0) tc_commit(sm.kv_empty + s);
      __syncwarp();
    };

    for (int j = 0; ok && j <= st.n; ++j) {
      if (C::kAliasP) {
        if (j >= 1) do_pv(j - 1);
        if (ok && j < st.n) do_s(j);
      } else {
        if (j < st.n) do_s(j);
        if (ok && j >= 1) do_pv(j - 1);
      }
    }
    ring = ring0 + 2u * st.n;
  }
  // Wait for every MMA this warp issued before the CTA frees TMEM.
  if (lane == 0) {
    tc_commit(sm.drain);
    drain_bar(sm.drain, 0);
  }
  __syncwarp();
}

template <int D>
__device__ void softmax_role(const TcParams& p, const Smem<D>& sm, const Ctl& ctl, uint32_t tmem, int X) {
  using C = Cfg<D>;
  const int row = threadIdx.x & 127;
  const uint32_t lane_off = (uint32_t)(((threadIdx.x >> 5) & 3) * 32) << 16;
  const uint32_t tS = tmem + C::s_col(X) + lane_off;
  const uint32_t tP = tmem + C::p_col(X) + lane_off;
  const uint32_t tO = tmem + C::o_col(X) + lane_off;
  const float sl2 = p.scale_log2;
  uint32_t s_seen = 0, pv_base = 0;
  bool ok = true;
  for (int64_t it = blockIdx.x; ok && it < p.n_items; it += gridDim.x) {
    const WorkItem w = p.items[it];
    if (X >= w.n_q) continue;
    const Stream st(w);
    const int nX = st.count(X);
    float m = -INFINITY, l = 0.f;
    for (int t = 0; t < nX; ++t) {
      const int valid = st.valid(w, X, t);
      ok = wait_bar(sm.s_full + X, s_seen & 1, ctl);
      if (!ok) break;
      ++s_seen;
      tc_fence_after();
      uint32_t sr[128];
      tmem_ld128(tS, sr);
      if (!C::kAliasP) {
        tc_fence_before();
        mbar_arrive(sm.s_free + X);
      }
      float s[128];
#pragma unroll
      for (int c = 0; c < 128; ++c) s[c] = __uint_as_float(sr[c]);
      if (valid < kTileN) {
#pragma unroll
        for (int c = 0; c < 128; ++c) s[c] = c < valid ? s[c] : -INFINITY;
      }
      float mx0 = s[0], mx1 = s[1], mx2 = s[2], mx3 = s[3];
#pragma unroll
      for (int c = 4; c < 128; c += 4) {
        mx0 = fmaxf(mx0, s[c]);
        mx1 = fmaxf(mx1, s[c + 1]);
        mx2 = fmaxf(mx2, s[c + 2]);
        mx3 = fmaxf(mx3, s[c + 3]);
      }
      const float tile_m = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3)) * sl2;
      float m_new = m;
      if (t == 0) m_new = tile_m;
      else if (tile_m > m + kRescaleThreshold) m_new = tile_m;
      const bool resc = t > 0 && m_new != m;
      if (__any_sync(0xffffffffu, resc)) {
        // O holds the previous tiles' sum: wait for the last PV, then rescale in place.
        ok = wait_bar(sm.pv_done + X, (pv_base + t - 1) & 1, ctl);
        if (!ok) break;
        tc_fence_after();
        const float alpha = resc ? ex2(m - m_new) : 1.f;
        l *= alpha;
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(tO + 32 * c, o);
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
          tmem_st32(tO + 32 * c, o);
        }
        tmem_st_wait();
      }
      m = m_new;
      const float nm = -m;
      float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
      for (int c = 0; c < 128; c += 4) {
        s[c] = ex2(fmaf(s[c], sl2, nm));
        s[c + 1] = ex2(fmaf(s[c + 1], sl2, nm));
        s[c + 2] = ex2(fmaf(s[c + 2], sl2, nm));
        s[c + 3] = ex2(fmaf(s[c + 3], sl2, nm));
        a0 += s[c];
        a1 += s[c + 1];
        a2 += s[c + 2];
        a3 += s[c + 3];
      }
      l += (a0 + a1) + (a2 + a3);
      if (!C::kAliasP && t > 0) {
        // Separate P columns: the previous P must have been consumed.
        ok = wait_bar(sm.pv_done + X, (pv_base + t - 1) & 1, ctl);
        if (!ok) break;
        tc_fence_after();
      }
      uint32_t pk[32];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
#pragma unroll
        for (int i = 0; i < 32; ++i) pk[i] = pack_bf16x2(s[64 * h + 2 * i], s[64 * h + 2 * i + 1]);
        tmem_st32(tP + 32 * h, pk);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(sm.p_full + X);
    }
    if (!ok) break;
    // Epilogue: O / l, 16-byte stores of this thread's row.
    ok = wait_bar(sm.pv_done + X, (pv_base + nX - 1) & 1, ctl);
    if (!ok) break;
    tc_fence_after();
    pv_base += nX;
    const int rows = X ? w.qB_rows : w.qA_rows;
    const int qrow = (X ? w.qB_row0 : w.qA_row0) + row;
    const bool live = row < rows;
    const float inv = 1.f / l;
    const float lse2 = m + __log2f(l);
    if (w.split_slot < 0) {
      __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(p.out) + ((int64_t)qrow * p.H + w.head) * D;
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(tO + 32 * c, o);
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          pk[i] = pack_bf16x2(__uint_as_float(o[2 * i]) * inv, __uint_as_float(o[2 * i + 1]) * inv);
        if (live) {
          uint4* d4 = reinterpret_cast<uint4*>(dst + 32 * c);
#pragma unroll
          for (int i = 0; i < 4; ++i) d4[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
        }
      }
      if (live && p.lse) p.lse[(int64_t)w.head * p.T_suf + qrow] = lse2 * 0.69314718055994531f;
    } else {
      const int64_t slot = w.split_slot + X;
      float* dst = p.part_o + (slot * kTileM + row) * D;
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(tO + 32 * c, o);
        if (live) {
          float4* d4 = reinterpret_cast<float4*>(dst + 32 * c);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            d4[i] = make_float4(__uint_as_float(o[4 * i]) * inv, __uint_as_float(o[4 * i + 1]) * inv,
                                __uint_as_float(o[4 * i + 2]) * inv, __uint_as_float(o[4 * i + 3]) * inv);
        }
      }
      if (live) p.part_lse[slot * kTileM + row] = lse2;
    }
  }
}

template <int D>
__global__ void __launch_bounds__(kTcThreads, 1) bat_attn_tc_kernel(const __grid_constant__ TcParams p) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Smem<D> sm;
  sm.q = base;
  sm.kv = base + 2 * C::kTileBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm.kv + C::kStages * C::kTileBytes);
  sm.kv_full = bars;
  sm.kv_empty = bars + C::kStages;
  sm.q_full = sm.kv_empty + C::kStages;
  sm.q_empty = sm.q_full + 2;
  sm.s_full = sm.q_empty + 2;
  sm.s_free = sm.s_full + 2;
  sm.p_full = sm.s_free + 2;
  sm.pv_done = sm.p_full + 2;
  sm.drain = sm.pv_done + 2;
  sm.tmem_slot = reinterpret_cast<uint32_t*>(sm.drain + 1);
  sm.abort_flag = reinterpret_cast<volatile int*>(sm.tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(sm.kv_full + s, 1);
      mbar_init(sm.kv_empty + s, 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(sm.q_full + x, 1);
      mbar_init(sm.q_empty + x, 1);
      mbar_init(sm.s_full + x, 1);
      mbar_init(sm.s_free + x, 128);
      mbar_init(sm.p_full + x, 128);
      mbar_init(sm.pv_done + x, 1);
    }
    mbar_init(sm.drain, 1);
    *sm.abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 8 && (threadIdx.x & 31) == 0) {
    prefetch_tmap(&p.tm_q);
    prefetch_tmap(&p.tm_ks);
    prefetch_tmap(&p.tm_vs);
    prefetch_tmap(&p.tm_kc);
    prefetch_tmap(&p.tm_vc);
  }
  if (warp == 9) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(sm.tmem_slot)),
                 "r"(C::kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *sm.tmem_slot;
  const Ctl ctl{sm.abort_flag, p.status, p.wait_ns};

  if (warp == 8) producer_role<D>(p, sm, ctl);
  else if (warp == 9) mma_role<D>(p, sm, ctl, tmem);
  else softmax_role<D>(p, sm, ctl, tmem, warp >> 2);

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 9)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(C::kTmemCols) : "memory");
}

}  // namespace

size_t attn_tc_smem_bytes(int d) { return d == 128 ? Cfg<128>::kSmemBytes : Cfg<64>::kSmemBytes; }

cudaError_t launch_attn_tc(int d, const TcParams& p, int grid, cudaStream_t s) {
  if (grid <= 0) return cudaSuccess;
  if (d == 128) {
    static bool attr = false;   // per process; the attribute is per function, not per device
    cudaError_t e = cudaFuncSetAttribute(bat_attn_tc_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)Cfg<128>::kSmemBytes);
    if (e != cudaSuccess) return e;
    (void)attr;
    bat_attn_tc_kernel<128><<<grid, kTcThreads, Cfg<128>::kSmemBytes, s>>>(p);
  } else if (d == 64) {
    cudaError_t e = cudaFuncSetAttribute(bat_attn_tc_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)Cfg<64>::kSmemBytes);
    if (e != cudaSuccess) return e;
    bat_attn_tc_kernel<64><<<grid, kTcThreads, Cfg<64>::kSmemBytes, s>>>(p);
  } else {
    return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t device_status_word(uint32_t** out) {
  return cudaGetSymbolAddress(reinterpret_cast<void**>(out), g_status_word);
}

}  // namespace bat
