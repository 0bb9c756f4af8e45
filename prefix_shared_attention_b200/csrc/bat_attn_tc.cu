// Bipartite prefix-shared attention forward on tcgen05 tensor cores (sm_100a).
//
// Operation (Bat lead page, sections "This paper's idea" and "Why it works"): each
// request's suffix rows attend, with no mask, over [cached prefix K/V ; own suffix K/V].
// The prefix K/V is computed once and cached; every request that references it reuses it.
//
// One persistent CTA per SM takes work items from the list built by the host grouping pass,
// in list order from a global counter (so the items of one prefix group run at the same time
// on neighbouring SMs and share their K/V tiles through L2).  A work item holds one head and
// up to two 128-row query tiles (A, B) that read the same prefix.
// The CTA streams the item's key tiles through shared memory with TMA, once each, and both
// query tiles consume every shared tile:
//
//   warp 8       TMA producer: takes the work items; Q tiles and the K tiles (d = 128) into a K
//                ring, or (d = 64) the K and V tiles into one ring in the order the MMA
//                issuers consume them: K0, K1, V0, K2, V1, ... (the K tile of key tile j+1
//                ahead of the V tile of j)
//   warps 9, 10  MMA issuers (one lane each) of tiles A and B: S = Q.K^T (SS), O += P.V
//                (d = 128: SS, P read from shared memory; d = 64: TS, P read from TMEM).  S of
//                key tile j+1 is issued as soon as the softmax has read S of tile j, so it is
//                computed while the softmax of tile j runs; PV of tile j follows its P (at
//                d = 64 in two 64-key halves, each as soon as its half of P is written).
//   warp 11      d = 128: TMA producer of the V tiles into a V ring; d = 64: TMA producer of
//                the Q tiles (so the K/V producer streams across item boundaries)
//   warps 0..3   softmax + epilogue of tile A (one thread per query row = TMEM lane); the
//                epilogue writes O / l through shared memory with bulk tensor stores
//   warps 4..7   softmax + epilogue of tile B
//
// TMEM (512 columns): S_A, S_B (128 fp32 columns each), O_A, O_B (d columns each); at d = 64
// P (bf16 pairs, 64 columns per tile) takes the remaining 128 columns, at d = 128 P lives in
// shared memory (one 32 KiB tile per query tile) because TMEM is full.
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

// A compile-time bool as a type (selects one of the two compiled copies of the softmax tile).
template <bool B>
struct BoolC {
  static constexpr bool value = B;
};

// Status words of this device: [0] bit 0 a wait timed out, bit 1 a debug check failed;
// [1], [2] the first failed debug check and its value.
__device__ uint32_t g_status_word[4];

// Compile-time event trace of CTA 0 (off unless built with -DBAT_TRACE): per role, a list of
// (code, clock64) pairs; code = event | x << 8 | index << 16.
#ifdef BAT_TRACE
constexpr int kTraceCap = 8192;
__device__ unsigned long long* g_trace;   // [7 roles][kTraceCap][2]
// The buffer pointer is read once per role (a global load per event would itself stall the
// traced warp by an L2 round trip).
__device__ __forceinline__ unsigned long long* trace_base(int role) {
  return (blockIdx.x == 0 && (threadIdx.x & 31) == 0 && g_trace) ? g_trace + (size_t)role * kTraceCap * 2 : nullptr;
}
__device__ __forceinline__ void trace(unsigned long long* tp, int& n, uint32_t ev, uint32_t x, uint32_t idx) {
  if (tp && n < kTraceCap) {
    const unsigned long long c = clock64();
    tp[2 * n] = ev | (x << 8) | (idx << 16);
    tp[2 * n + 1] = c;
    ++n;
  }
}
#define BAT_TRACE_INIT(role) unsigned long long* trace_p = trace_base(role)
#define BAT_TRACE_EV(role, n, ev, x, idx) trace(trace_p, n, ev, x, idx)
#define BAT_PHASE_FLUSH() ((void)0)
#elif defined(BAT_PHASE)
// Compile-time phase profile (off unless built with -DBAT_PHASE): every warp accumulates, per
// trace event code, the clocks since its previous event in registers and writes the totals
// once at the end ([grid][12 warps][20] words), so the profile barely perturbs the timing.
__device__ unsigned* g_phase;
#define BAT_TRACE_INIT(role)                                                  \
  uint32_t ph_acc[20];                                                        \
  _Pragma("unroll") for (int ph_i = 0; ph_i < 20; ++ph_i) ph_acc[ph_i] = 0; \
  uint32_t ph_last = (uint32_t)clock64()
#define BAT_TRACE_EV(role, n, ev, x, idx)      \
  do {                                         \
    const uint32_t ph_c = (uint32_t)clock64(); \
    ph_acc[ev] += ph_c - ph_last;              \
    ph_last = ph_c;                            \
  } while (0)
#define BAT_PHASE_FLUSH()                                                                 \
  do {                                                                                    \
    if (g_phase && (threadIdx.x & 31) == 0) {                                             \
      unsigned* ph_o = g_phase + ((size_t)blockIdx.x * 12 + (threadIdx.x >> 5)) * 20;     \
      _Pragma("unroll") for (int ph_i = 0; ph_i < 20; ++ph_i) ph_o[ph_i] = ph_acc[ph_i]; \
    }                                                                                     \
  } while (0)
#else
#define BAT_TRACE_INIT(role) ((void)0)
#define BAT_TRACE_EV(role, n, ev, x, idx) ((void)0)
#define BAT_PHASE_FLUSH() ((void)0)
#endif

constexpr float kRescaleThreshold = 8.0f;   // log2 units: P stays <= 2^8 between rescales
constexpr int kItemQ = 4;                   // work items the producer may run ahead by
constexpr uint64_t kDrainNs = 200ull * 1000 * 1000;

#include "bat_ptx.h"

// ------------------------------------------------------------------------------------
// Compile-time layout

template <int D>
struct Cfg {
  static constexpr int kPanels = D / 64;                 // 64-element (128-byte) column panels
  static constexpr int kPanelBytes = kTileM * 128;       // 128 rows x 128 bytes
  static constexpr int kTileBytes = kPanels * kPanelBytes;
  // P in shared memory at d = 128 (TMEM is full); at d = 64 it stays in TMEM (P in shared memory
  // there, with the ring cut from 10 to 8 stages, measured 8 % slower on item-as-prefix).
  static constexpr bool kPSmem = D == 128;
  // One P buffer per query tile: a P tile (128 rows x 128 keys, bf16) when P lives in shared
  // memory, else only the output staging tile (128 rows x d).
  static constexpr int kPTileBytes = kPSmem ? 2 * kPanelBytes : kTileBytes;
  // One shared-memory tile per query tile: P (d = 128), and at the end of an item the staging
  // buffer of the output tile (both d).
  static constexpr int kPBufs = 2;
  // K/V ring depth (fills 227 KB).  d = 128: three tiles, split into a K ring of two and a V
  // ring of one, each with its own producer warp, so a K tile is never queued behind a V tile
  // (measured 1-2% faster than one shared ring of three).  d = 64: one ring of ten, filled in
  // consumption order by one producer (every split of it measured slower).
  static constexpr bool kTwoRings = D == 128;
  static constexpr int kStages = D == 128 ? 3 : 10;
  static constexpr int kStagesK = kTwoRings ? 2 : kStages;
  static constexpr int kStagesV = kStages - kStagesK;
  // Q tiles: loaded by warp 11 when it is not the V producer (d = 64), so the K/V producer never
  // waits for the next item's Q buffer to free and keeps streaming K/V tiles across item
  // boundaries; at d = 128 the K producer loads them.
  static constexpr bool kQWarp = !kTwoRings;
  // Warps that pop every work item: 8 softmax, 2 MMA issuers and warp 11 (V or Q producer).
  static constexpr int kItemConsumers = 11;
  // d = 64: PV is issued in two halves of 64 keys, each as soon as the softmax has written that
  // half of P, so the next tile's P can overwrite the first half early (measured faster at
  // d = 64, slower at d = 128, where one PV per tile and one P hand-off are issued instead).
  static constexpr int kPVHalves = D == 64 ? 2 : 1;
  static constexpr uint32_t kTmemCols = 512;
  __host__ __device__ static constexpr uint32_t s_col(int x) { return 128u * x; }
  __host__ __device__ static constexpr uint32_t o_col(int x) { return 256u + (uint32_t)D * x; }
  __host__ __device__ static constexpr uint32_t p_col(int x) { return 384u + 64u * x; }   // d = 64 only
  static constexpr uint32_t kIdescS = make_idesc(128, 128, false);
  static constexpr uint32_t kIdescSHalf = make_idesc(128, 64, false);   // key tiles of <= 64 valid keys
  // d = 64: a key tile with at most 64 valid keys (a short prefix, the ragged end of a stream)
  // gets S at N = 64, PV over its first 64 keys and no exponentials or P stores for the masked
  // half (measured +4 % on item-as-prefix, whose prefixes are 32 keys long).  At d = 128 the
  // same skip made the full-tile softmax slower, so it is off there.
  static constexpr bool kHalfSkip = D == 64;
  static constexpr uint32_t kIdescPV = make_idesc(128, D, true);
  static constexpr int kBarBytes = 8 * (3 * kStages + 2 * 4 + 4 * 2 + 2 + 2 * kItemQ) + 16 + 4 * kItemQ;
  static constexpr size_t kSmemBytes =
      1024 + (size_t)(2 + kStages) * kTileBytes + (size_t)kPBufs * kPTileBytes + kBarBytes;
  static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
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
  // Valid keys in global tile j (the rest of the tile belongs to other rows: masked).
  __device__ __forceinline__ int tile_valid(const WorkItem& w, int j) const {
    if (j < npre) return min(kTileN, w.pre_len - j * kTileN);
    const int k = j - npre;
    if (shared) return min(kTileN, w.sA_len - k * kTileN);
    const int mm = nsA < nsB ? nsA : nsB;
    const int x = k < 2 * mm ? (k & 1) : (nsA > nsB ? 0 : 1);
    const int idx = k < 2 * mm ? (k >> 1) : mm + (k - 2 * mm);
    return min(kTileN, (x ? w.sB_len : w.sA_len) - idx * kTileN);
  }
  // Ring position pos (0 .. 2n-1) of the item's K/V loads: K0, K1, V0, K2, V1, ..., K(n-1),
  // V(n-2), V(n-1).  This is the order in which each MMA issuer uses them (S of key tile j+1,
  // then PV of key tile j), so every issuer walks the ring strictly in order.
  __device__ __forceinline__ void slot(int pos, int& j, bool& is_v) const {
    if (pos == 0) {
      j = 0;
      is_v = false;
    } else if (pos == 2 * n - 1) {
      j = n - 1;
      is_v = true;
    } else if (pos & 1) {
      j = (pos + 1) >> 1;
      is_v = false;
    } else {
      j = (pos >> 1) - 1;
      is_v = true;
    }
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
    // One suspension never outlasts the wait's own limit (1 ms at most).
    const uint32_t hint = c.limit_ns < 1000000ull ? (uint32_t)c.limit_ns : 1000000u;
    while (true) {
      ok = mbar_test_suspend(bar, parity, hint);
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
  uint8_t* p;        // [kPBufs][kPTileBytes]: P of tiles A, B (when in shared memory) / output staging
  uint8_t* kv;       // [kStages][kTileBytes]: the K ring (or the shared ring), then the V ring
  uint64_t* kv_full;   // [kStages]
  uint64_t* kv_empty;  // [kStages]
  uint64_t* q_full;   // [2]
  uint64_t* q_empty;  // [2]
  uint64_t* s_full;   // [2]
  uint64_t* s_free;   // [2]
  uint64_t* p_full;   // [2][2]: P of tile x, keys 64h .. 64h+63 written
  uint64_t* pv_done;  // [2][2]: PV of tile x over keys 64h .. 64h+63 done
  uint64_t* drain;    // [2]
  uint64_t* v_zeroed;  // [kStages]: the tail rows of a ragged V tile in this slot are zeroed
  uint64_t* itq_full;   // [kItemQ]
  uint64_t* itq_empty;  // [kItemQ]
  volatile int* itq;    // [kItemQ] work-item indices handed from the producer to the others
  uint32_t* tmem_slot;
  volatile int* abort_flag;
};

// Work items are handed out dynamically (a global counter), so items next to each other in
// the list (same prefix group, same head) run at the same time on different CTAs and share
// their prefix and suffix tiles through L2.  The producer warp takes the next index and
// passes it to the MMA and softmax warps through a small queue; -1 ends the kernel.
template <int D>
__device__ __forceinline__ int pop_item(const Smem<D>& sm, uint32_t& k, const Ctl& ctl, bool& ok) {
  const uint32_t slot = k % kItemQ;
  ok = wait_bar(sm.itq_full + slot, (k / kItemQ) & 1, ctl);
  const int it = ok ? sm.itq[slot] : -1;
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(sm.itq_empty + slot);
  ++k;
  return it;
}

// ------------------------------------------------------------------------------------
// Roles

// The rings of K/V tiles: the K ring and the V ring (two producers), or one ring that holds
// both in consumption order (one producer).  Slot of ring sequence number r: first(R) + r % depth(R).
enum Ring { kRingK = 0, kRingV = 1, kRingKV = 2 };
template <int D, int R>
struct RingGeom {
  static constexpr uint32_t kDepth = R == kRingK ? Cfg<D>::kStagesK : R == kRingV ? Cfg<D>::kStagesV : Cfg<D>::kStages;
  static constexpr uint32_t kFirst = R == kRingV ? Cfg<D>::kStagesK : 0;
};

// Loads one item's tiles of ring R, in the order the MMA issuers consume them; `ring` counts
// the loads this warp has issued into R.  Returns false on abort.
template <int D, int R>
__device__ __forceinline__ bool load_ring(const TcParams& p, const Smem<D>& sm, const Ctl& ctl, const WorkItem& w,
                                          const Stream& st, uint32_t& ring, int& trace_n) {
  (void)trace_n;
  using C = Cfg<D>;
  using G = RingGeom<D, R>;
  const int lane = threadIdx.x & 31;
  const int npos = R == kRingKV ? 2 * st.n : st.n;
#ifdef BAT_TRACE
  BAT_TRACE_INIT(R == kRingV ? 6 : 5);   // load events of the K (or shared) ring and of the V ring
#endif
  for (int pos = 0; pos < npos; ++pos) {
    int j = pos, mask, row0;
    bool is_v = R == kRingV, from_cache;
    if (R == kRingKV) st.slot(pos, j, is_v);
    st.tile(w, j, mask, from_cache, row0);
    const uint32_t s = G::kFirst + ring % G::kDepth, ph = (ring / G::kDepth) & 1;
    if (!wait_bar(sm.kv_empty + s, ph ^ 1, ctl)) return false;
    if (lane == 0) {
      const CUtensorMap* m = from_cache ? (is_v ? &p.tm_vc : &p.tm_kc) : (is_v ? &p.tm_vs : &p.tm_ks);
      int y = row0, x = w.head * D;
      if (!BAT_DCHECK(p.status, y >= 0 && y < (from_cache ? (p.T_cache - p.chk_shrink) : (p.T_suf - p.chk_shrink)) && x >= 0 && x + D <= p.H * D,
                      from_cache ? kChkCacheLoad : kChkSufLoad, y))
        y = x = 0;
      mbar_expect_tx(sm.kv_full + s, C::kTileBytes);
#pragma unroll
      for (int pn = 0; pn < C::kPanels; ++pn)
        tma_load_2d(sm.kv + s * C::kTileBytes + pn * C::kPanelBytes, m, x + pn * 64, y, sm.kv_full + s);
    }
#ifdef BAT_TRACE
    BAT_TRACE_EV(0, trace_n, 3, is_v ? 1 : 0, ring);
#endif
    __syncwarp();
    ++ring;
  }
  return true;
}

// After an abort: waits (bounded) for the last loads issued into ring R to land.
template <int D, int R>
__device__ __forceinline__ void drain_ring(const Smem<D>& sm, uint32_t ring) {
  using G = RingGeom<D, R>;
  const uint32_t n = ring < G::kDepth ? ring : G::kDepth;
  for (uint32_t i = ring - n; i < ring; ++i) drain_bar(sm.kv_full + G::kFirst + i % G::kDepth, (i / G::kDepth) & 1);
}

template <int D>
__device__ void producer_role(const TcParams& p, const Smem<D>& sm, const Ctl& ctl) {
  using C = Cfg<D>;
  const int lane = threadIdx.x & 31;
  uint32_t ring = 0, qcnt[2] = {0, 0}, kq = 0;
  bool ok = true;
  int tn = 0, ring_tn = 0;
  (void)tn;
  BAT_TRACE_INIT(0);
  while (ok) {
    const uint32_t slot = kq % kItemQ;
    ok = wait_bar(sm.itq_empty + slot, ((kq / kItemQ) & 1) ^ 1, ctl);
    if (!ok) break;
    int it = 0;
    if (lane == 0) it = atomicAdd(p.item_counter, 1);
    it = __shfl_sync(0xffffffffu, it, 0);
    const bool done = it >= p.n_items;
    if (lane == 0) {
      sm.itq[slot] = done ? -1 : it;
      mbar_arrive(sm.itq_full + slot);
    }
    __syncwarp();
    ++kq;
    if (done) break;
    const WorkItem w = p.items[it];
    if (lane == 0) {
      // The item's fields stay inside the tensors (debug builds; the accesses are checked too).
      BAT_DCHECK(p.status,
                 w.head >= 0 && w.head < p.H && (w.n_q == 1 || w.n_q == 2) && w.qA_rows >= 1 && w.qA_rows <= kTileM &&
                     w.qA_row0 >= 0 && w.qA_row0 + w.qA_rows <= (p.T_suf - p.chk_shrink) && w.sA_row0 >= 0 &&
                     w.sA_row0 + w.sA_len <= (p.T_suf - p.chk_shrink) && w.pre_len >= 0 &&
                     (w.pre_len == 0 || (w.pre_row0 >= 0 && w.pre_row0 + w.pre_len <= (p.T_cache - p.chk_shrink))) &&
                     (w.n_q == 1 || (w.qB_rows >= 1 && w.qB_rows <= kTileM && w.qB_row0 >= 0 &&
                                     w.qB_row0 + w.qB_rows <= (p.T_suf - p.chk_shrink) && w.sB_row0 >= 0 &&
                                     w.sB_row0 + w.sB_len <= (p.T_suf - p.chk_shrink))) &&
                     (w.split_slot < 0 || w.split_slot + w.n_q <= p.n_slots),
                 kChkItem, it);
    }
    BAT_TRACE_EV(0, tn, 1, 0, kq);
    for (int x = 0; ok && !C::kQWarp && x < w.n_q; ++x) {
      ok = wait_bar(sm.q_empty + x, (qcnt[x] & 1) ^ 1, ctl);
      if (!ok) break;
      BAT_TRACE_EV(0, tn, 2, x, kq);
      if (lane == 0) {
        int y = x ? w.qB_row0 : w.qA_row0, cx = w.head * D;
        if (!BAT_DCHECK(p.status, y >= 0 && y < (p.T_suf - p.chk_shrink) && cx >= 0 && cx + D <= p.H * D, kChkQLoad, y)) y = cx = 0;
        mbar_expect_tx(sm.q_full + x, C::kTileBytes);
#pragma unroll
        for (int pn = 0; pn < C::kPanels; ++pn)
          tma_load_2d(sm.q + x * C::kTileBytes + pn * C::kPanelBytes, &p.tm_q, cx + pn * 64, y, sm.q_full + x);
      }
      __syncwarp();
      ++qcnt[x];
    }
    const Stream st(w);
    ok = load_ring<D, C::kTwoRings ? kRingK : kRingKV>(p, sm, ctl, w, st, ring, ring_tn);
  }
  BAT_PHASE_FLUSH();
  if (!ok && lane == 0) {
    // Let every copy this warp issued land before the CTA releases its shared memory.
    drain_ring<D, C::kTwoRings ? kRingK : kRingKV>(sm, ring);
    for (int x = 0; x < 2; ++x)
      if (qcnt[x]) drain_bar(sm.q_full + x, (qcnt[x] - 1) & 1);
  }
  __syncwarp();
}

// Q producer (warp 11, d = 64): the query tiles of every item into the two Q buffers, each as
// soon as the previous item's last S has read that buffer.  It pops the same work items as
// every other role.
template <int D>
__device__ void qproducer_role(const TcParams& p, const Smem<D>& sm, const Ctl& ctl) {
  using C = Cfg<D>;
  const int lane = threadIdx.x & 31;
  uint32_t qcnt[2] = {0, 0}, kq = 0;
  bool ok = true;
  while (ok) {
    const int it = pop_item<D>(sm, kq, ctl, ok);
    if (it < 0) break;
    const WorkItem w = p.items[it];
    for (int x = 0; ok && x < w.n_q; ++x) {
      ok = wait_bar(sm.q_empty + x, (qcnt[x] & 1) ^ 1, ctl);
      if (!ok) break;
      if (lane == 0) {
        int y = x ? w.qB_row0 : w.qA_row0, cx = w.head * D;
        if (!BAT_DCHECK(p.status, y >= 0 && y < (p.T_suf - p.chk_shrink) && cx >= 0 && cx + D <= p.H * D, kChkQLoad, y))
          y = cx = 0;
        mbar_expect_tx(sm.q_full + x, C::kTileBytes);
#pragma unroll
        for (int pn = 0; pn < C::kPanels; ++pn)
          tma_load_2d(sm.q + x * C::kTileBytes + pn * C::kPanelBytes, &p.tm_q, cx + pn * 64, y, sm.q_full + x);
      }
      __syncwarp();
      ++qcnt[x];
    }
  }
  if (!ok && lane == 0) {
    for (int x = 0; x < 2; ++x)
      if (qcnt[x]) drain_bar(sm.q_full + x, (qcnt[x] - 1) & 1);
  }
  __syncwarp();
}

// V producer (warp 11, d = 128): the value tiles of every item, in key-tile order, into the
// V ring.  It pops the same work items as every other role.
template <int D>
__device__ void vproducer_role(const TcParams& p, const Smem<D>& sm, const Ctl& ctl) {
  const int lane = threadIdx.x & 31;
  uint32_t ring = 0, kq = 0;
  bool ok = true;
  int ring_tn = 0;
  while (ok) {
    const int it = pop_item<D>(sm, kq, ctl, ok);
    if (it < 0) break;
    const WorkItem w = p.items[it];
    const Stream st(w);
    ok = load_ring<D, kRingV>(p, sm, ctl, w, st, ring, ring_tn);
  }
  if (!ok && lane == 0) drain_ring<D, kRingV>(sm, ring);
  __syncwarp();
}

// Zeroes rows [valid, valid rounded up to 16) of a K/V tile in shared memory, in every
// 64-column panel (one warp).  The 128-byte swizzle only permutes the 16-byte chunks within a
// row, so a whole row is the same 128 bytes with or without it.  The writes are made visible
// to the tensor core (async proxy) before the warp leaves.
template <int D>
__device__ __forceinline__ void zero_tail_rows(uint8_t* tile, int valid) {
  using C = Cfg<D>;
  const int lane = threadIdx.x & 31;
  const int n = (((valid + 15) & ~15) - valid) * C::kPanels * 8;   // 16-byte chunks
  const uint32_t base = smem_u32(tile) + (uint32_t)valid * 128;
  for (int i = lane; i < n; i += 32) {
    const int rp = i >> 3;   // (row - valid) * kPanels + panel
    st_shared_v4(base + (rp % C::kPanels) * C::kPanelBytes + (rp / C::kPanels) * 128 + (i & 7) * 16, 0u, 0u, 0u, 0u);
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  __syncwarp();
}

// MMA issuer of query tile X (warp 9 for A, warp 10 for B).  A single issuing thread would
// serialise both tiles' bookkeeping against a tensor-core queue only about one instruction
// deep; with one issuer per tile, one tile's waits and commits overlap the other's MMAs.
// tcgen05.commit tracks only the committing thread's MMAs, so every K/V slot is released by
// two arrivals, one per issuer: a commit after its MMAs read the slot, or, for a tile this
// query tile does not read, a plain arrive once the tile has landed.
//
// Each issuer takes the tiles in one order (K0, K1, V0, K2, V1, ...), which is also the order
// of the shared ring and the order of each of the two rings: S of key tile j+1 waits only for
// the softmax to have read S of tile j (S has its own TMEM columns), so it is computed while
// that softmax runs; PV of tile j waits for its P.  Every wait is on the issuer's next tile or
// on its own softmax, which only needs earlier tiles, and every slot is freed by tiles earlier
// in that order, so no ring depth can deadlock (with two rings the producers also share only
// the work-item queue, which they both pop in order).
template <int D>
__device__ void mma_role(const TcParams& p, const Smem<D>& sm, const Ctl& ctl, uint32_t tmem, int X) {
  using C = Cfg<D>;
  const int lane = threadIdx.x & 31;
  uint32_t ring = 0, vring = 0, qcnt = 0, s_issued = 0, p_seen = 0;
  uint32_t vz_par = 0;   // bit s: parity of the next v_zeroed phase of ring slot s
  bool ok = true;
  int tn = 0;
  (void)tn;
  BAT_TRACE_INIT(1 + X);
  // Descriptors are computed once; per instruction only a constant is added to the start
  // address field (addresses stay below 256 KiB, so the 14-bit field never carries).
  const uint64_t qdesc = sdesc_sw128(smem_u32(sm.q) + X * C::kTileBytes, 16, 1024);
  const uint64_t pdesc = sdesc_sw128(smem_u32(sm.p) + X * C::kPTileBytes, 16, 1024);
  const uint64_t kdesc0 = sdesc_sw128(smem_u32(sm.kv), 16, 1024);
  const uint64_t vdesc0 = sdesc_sw128(smem_u32(sm.kv), C::kPanelBytes, 1024);
  const uint32_t s_t = tmem + C::s_col(X), o_t = tmem + C::o_col(X), p_t = tmem + C::p_col(X);

  uint32_t kq = 0;
  while (ok) {
    const int it = pop_item<D>(sm, kq, ctl, ok);
    if (it < 0) break;
    const WorkItem w = p.items[it];
    const Stream st(w);
    // Sequence numbers of the item's first K and V tiles in their rings (one shared ring at
    // d = 64, where the item's position pos is its sequence number).
    const uint32_t kr0 = ring, vr0 = vring;
    if constexpr (C::kTwoRings) {
      ring += (uint32_t)st.n;
      vring += (uint32_t)st.n;
    } else {
      ring += 2u * st.n;
    }
    const bool mine = X < w.n_q;
    int s_left = mine ? st.count(X) : 0;
    bool first_s = true, first_pv = true;
    for (int pos = 0; ok && pos < 2 * st.n; ++pos) {
      int j, mask, row0;
      bool is_v, from_cache;
      st.slot(pos, j, is_v);
      st.tile(w, j, mask, from_cache, row0);
      uint32_t s, ph;
      if constexpr (C::kTwoRings) {
        const uint32_t r = (is_v ? vr0 : kr0) + j;
        s = is_v ? RingGeom<D, kRingV>::kFirst + r % C::kStagesV : r % C::kStagesK;
        ph = (r / (is_v ? C::kStagesV : C::kStagesK)) & 1;
      } else {
        const uint32_t r = kr0 + pos;
        s = r % C::kStages;
        ph = (r / C::kStages) & 1;
      }
      if (pos == 0) BAT_TRACE_EV(1 + X, tn, 6, X, s_issued);
#ifdef BAT_TRACE
      BAT_TRACE_EV(1 + X, tn, 8, is_v ? 1 : 0, C::kTwoRings ? (is_v ? vr0 + j : kr0 + j) : kr0 + pos);
#endif
      ok = wait_bar(sm.kv_full + s, ph, ctl);
      if (!ok) break;
      if (!mine || !((mask >> X) & 1)) {
        // A tile this query tile does not read: release the slot once it has landed.
        if (lane == 0) mbar_arrive(sm.kv_empty + s);
        __syncwarp();
        continue;
      }
      if (!is_v) {
        BAT_TRACE_EV(1 + X, tn, 4, X, s_issued);
        if (first_s) {
          ok = wait_bar(sm.q_full + X, qcnt & 1, ctl);
          ++qcnt;
          first_s = false;
          BAT_TRACE_EV(1 + X, tn, 7, X, s_issued);
        }
        // The softmax must have read the previous S out of these columns.
        if (ok && s_issued > 0) ok = wait_bar(sm.s_free + X, (s_issued - 1) & 1, ctl);
        if (!ok) break;
        tc_fence_after();
        const uint64_t kd = kdesc0 + (uint64_t)((s * C::kTileBytes) >> 4);
        // A key tile with at most 64 valid keys: S over its first 64 keys only (the softmax
        // masks the other columns).
        const uint32_t idS = (C::kHalfSkip && st.tile_valid(w, j) <= 64) ? C::kIdescSHalf : C::kIdescS;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t off = (uint64_t)(((kk >> 2) * C::kPanelBytes + (kk & 3) * 32) >> 4);
          mma_ss_w(s_t, qdesc + off, kd + off, idS, kk > 0 ? 1u : 0u);
        }
        tc_commit_w(sm.s_full + X);
        if (s_left == 1) tc_commit_w(sm.q_empty + X);
        tc_commit_w(sm.kv_empty + s);
        --s_left;
        ++s_issued;
        BAT_TRACE_EV(1 + X, tn, 2, X, s_issued);
      } else {
        // O += P . V of key tile j, in kPVHalves parts (the part over keys 64h .. 64h+63 once the
        // softmax has written that half of P; with one part, the barriers of half 1 stand for
        // the whole tile).  16 keys per instruction = two 8-row swizzle groups of V (2 KiB); LBO
        // steps between V's 64-column panels.
        const uint64_t vd = vdesc0 + (uint64_t)((s * C::kTileBytes) >> 4);
        // PV runs only over the 16-key steps that hold a valid key.  P is exactly 0 beyond
        // `valid`, but the V rows there belong to other segments of the tensor (or were never
        // written), and 0 * NaN = NaN would poison the whole output row; so the steps past the
        // last valid key are not issued, and the rows between `valid` and the end of its
        // 16-key step are zeroed in shared memory by exactly one issuer: the lower-numbered
        // consumer of the tile, which the other consumer waits for.
        const int valid = st.tile_valid(w, j);
        const int kk_end = (valid + 15) >> 4;
        if (valid & 15) {
          if (X == ((mask & 1) ? 0 : 1)) {
            zero_tail_rows<D>(sm.kv + s * C::kTileBytes, valid);
            if (mask == 3 && lane == 0) mbar_arrive(sm.v_zeroed + s);
          } else {
            ok = wait_bar(sm.v_zeroed + s, (vz_par >> s) & 1, ctl);
            if (!ok) break;
          }
          if (mask == 3) vz_par ^= 1u << s;
        }
#pragma unroll
        for (int h = 2 - C::kPVHalves; h < 2; ++h) {
          BAT_TRACE_EV(1 + X, tn, 3, X, p_seen);
          ok = wait_bar(sm.p_full + 2 * X + h, p_seen & 1, ctl);
          if (!ok) break;
          tc_fence_after();
#pragma unroll
          for (int kk = C::kPVHalves == 2 ? 4 * h : 0; kk < 4 * h + 4; ++kk) {
            if (kk >= kk_end) break;
            const uint32_t acc = (first_pv && kk == 0) ? 0u : 1u;
            const uint64_t vk = vd + (uint64_t)(kk * 2048 / 16);
            if constexpr (C::kPSmem) {
              const uint64_t off = (uint64_t)(((kk >> 2) * C::kPanelBytes + (kk & 3) * 32) >> 4);
              mma_ss_w(o_t, pdesc + off, vk, C::kIdescPV, acc);
            } else {
              mma_ts_w(o_t, p_t + kk * 8, vk, C::kIdescPV, acc);
            }
          }
          tc_commit_w(sm.pv_done + 2 * X + h);
          BAT_TRACE_EV(1 + X, tn, 1, X, p_seen);
        }
        if (!ok) break;
        ++p_seen;
        tc_commit_w(sm.kv_empty + s);
        first_pv = false;
      }
      __syncwarp();
    }
  }
  BAT_PHASE_FLUSH();
  // Wait for every MMA this warp issued before the CTA frees TMEM.
  if (lane == 0) {
    tc_commit(sm.drain + X);
    drain_bar(sm.drain + X, 0);
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
  // d = 128: this thread's row of the P tile in shared memory (K-major, 128-byte swizzle:
  // 16-byte chunk c of row r sits at r * 128 + ((c ^ (r & 7)) << 4) within its 64-key panel).
  const uint32_t p_row = smem_u32(sm.p) + X * C::kPTileBytes + row * 128;
  const uint32_t p_sw = row & 7;
  const int wq = (threadIdx.x >> 5) & 3;           // this warp's 32-row group of the tile
  const uint32_t lane = threadIdx.x & 31;
  bool o_pending = false;                          // lane 0: a bulk store still reads this warp's P rows
  uint32_t s_seen = 0, pv_base = 0;
  bool ok = true;
  int tn = 0;
  (void)tn;
  BAT_TRACE_INIT(3 + X);
  uint32_t kq = 0;
  while (ok) {
    const int it = pop_item<D>(sm, kq, ctl, ok);
    if (it < 0) break;
    BAT_TRACE_EV(3 + X, tn, 15, X, s_seen);
    const WorkItem w = p.items[it];
    if (X >= w.n_q) continue;
    BAT_TRACE_EV(3 + X, tn, 16, X, s_seen);
    {
      if (o_pending) {
        // The previous item's output leaves this warp's P rows by a bulk store: it must have
        // read them before this item's P overwrites them.
        if (lane == 0) bulk_wait_read();
        __syncwarp();
        o_pending = false;
      }
    }
    const Stream st(w);
    const int nX = st.count(X);
    float m = -INFINITY, l = 0.f;
    for (int t = 0; t < nX; ++t) {
      const int valid = st.valid(w, X, t);
      ok = wait_bar(sm.s_full + X, s_seen & 1, ctl);
      if (!ok) break;
      BAT_TRACE_EV(3 + X, tn, 1, X, s_seen);
      ++s_seen;
      tc_fence_after();
      float s[128];
      tmem_ld128f(tS, s);
      BAT_TRACE_EV(3 + X, tn, 7, X, s_seen);
      // S is in registers: the issuer may compute the next S into these columns.
      tc_fence_before();
      mbar_arrive(sm.s_free + X);
      // The tile body; with kHalfSkip compiled twice: for full tiles and for tiles with at most
      // 64 valid keys.
      auto tile_body = [&](auto half_c) {
        constexpr bool HALF = decltype(half_c)::value;
        if (valid < kTileN) {
#pragma unroll
          for (int c = 0; c < 128; ++c) s[c] = c < valid ? s[c] : -INFINITY;
        }
        // Row maximum: eight independent 3-input-max chains (short dependency depth); four over
        // the first 64 columns for a tile with at most 64 valid keys.
        float mx[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          if (HALF && k >= 4) {
            mx[k] = -INFINITY;
            continue;
          }
          mx[k] = s[16 * k];
#pragma unroll
          for (int i = 1; i < 15; i += 2) mx[k] = max3f(mx[k], s[16 * k + i], s[16 * k + i + 1]);
          mx[k] = fmaxf(mx[k], s[16 * k + 15]);
        }
        const float tile_m = fmaxf(max3f(max3f(mx[0], mx[1], mx[2]), max3f(mx[3], mx[4], mx[5]), mx[6]), mx[7]) * sl2;
        float m_new = m;
        if (t == 0) m_new = tile_m;
        else if (tile_m > m + kRescaleThreshold) m_new = tile_m;
        const bool resc = t > 0 && m_new != m;
        if (__any_sync(0xffffffffu, resc)) {
          // O holds the previous tiles' sum: wait for the last PV, then rescale in place.
          ok = wait_bar(sm.pv_done + 2 * X + 1, (pv_base + t - 1) & 1, ctl);
          if (!ok) return;
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
        BAT_TRACE_EV(3 + X, tn, 8, X, s_seen);
        const float nm = -m;
        float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
        // Exponentials in two halves of 64 columns; each half is converted to bf16 pairs and
        // stored (TMEM or shared memory, asynchronously) while the next half's exponentials run.
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          // A tile with at most 64 valid keys: keys 64 .. 127 carry no weight and PV skips them,
          // so their exponentials and P stores are skipped (the barrier hand-offs stay).
          const bool skip = HALF && h == 1;
#pragma unroll
          for (int c = 64 * h; c < 64 * h + 64; c += 8) {
            if (skip) break;
#pragma unroll
            for (int k = 0; k < 8; k += 2) ffma2(s[c + k], s[c + k + 1], s[c + k], s[c + k + 1], sl2, nm);
#pragma unroll
            for (int k = 0; k < 8; ++k) s[c + k] = ex2(s[c + k]);
            fadd2(a0, a1, s[c], s[c + 1]);
            fadd2(a2, a3, s[c + 2], s[c + 3]);
            fadd2(a0, a1, s[c + 4], s[c + 5]);
            fadd2(a2, a3, s[c + 6], s[c + 7]);
          }
          if (t > 0 && (C::kPVHalves == 2 || h == 0)) {
            // This half of the previous P (with one PV part: all of it) must have been consumed
            // before it is overwritten.
            BAT_TRACE_EV(3 + X, tn, 12, X, s_seen);
            ok = wait_bar(sm.pv_done + 2 * X + (C::kPVHalves == 2 ? h : 1), (pv_base + t - 1) & 1, ctl);
            if (!ok) break;
            tc_fence_after();
            BAT_TRACE_EV(3 + X, tn, 11, X, s_seen);
          }
          uint32_t pk[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) pk[i] = pack_bf16x2(s[64 * h + 2 * i], s[64 * h + 2 * i + 1]);
          if (skip) {
          } else if constexpr (C::kPSmem) {
            // Keys 64h .. 64h+63 are panel h of the P tile.
#pragma unroll
            for (int cc = 0; cc < 8; ++cc)
              st_shared_v4(p_row + h * C::kPanelBytes + ((cc ^ p_sw) << 4), pk[4 * cc], pk[4 * cc + 1], pk[4 * cc + 2],
                           pk[4 * cc + 3]);
          } else {
            tmem_st32(tP + 32 * h, pk);
          }
          if (C::kPVHalves == 2 || h == 1) {
            if constexpr (C::kPSmem) {
              // Make the generic-proxy stores visible to the tensor core (async proxy).
              asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            } else {
              tmem_st_wait();
              tc_fence_before();
            }
            mbar_arrive(sm.p_full + 2 * X + h);
          }
        }
        if (!ok) return;
        l += (a0 + a1) + (a2 + a3);
      };
      if constexpr (C::kHalfSkip) {
        if (valid <= 64) tile_body(BoolC<true>{});
        else tile_body(BoolC<false>{});
      } else {
        tile_body(BoolC<false>{});
      }
      if (!ok) break;
      BAT_TRACE_EV(3 + X, tn, 2, X, s_seen);
    }
    if (!ok) break;
    // Epilogue: O / l, 16-byte stores of this thread's row.
    BAT_TRACE_EV(3 + X, tn, 5, X, s_seen);
    ok = wait_bar(sm.pv_done + 2 * X + 1, (pv_base + nX - 1) & 1, ctl);
    if (!ok) break;
    tc_fence_after();
    BAT_TRACE_EV(3 + X, tn, 13, X, s_seen);
    pv_base += nX;
    const int rows = X ? w.qB_rows : w.qA_rows;
    const int qrow = (X ? w.qB_row0 : w.qA_row0) + row;
    const bool live = row < rows;
    const float inv = 1.f / l;
    const float lse2 = m + __log2f(l);
    bool o_stored = false;
    {
      if (w.split_slot < 0 && rows >= 32 * (wq + 1)) {
        // All 32 rows of this warp belong to the request: O / l goes into the warp's rows of its
        // shared-memory tile (P at d = 128, free after the last PV; a staging tile at d = 64)
        // in the 128-byte-swizzled layout, then one bulk tensor store per 64-column panel
        // writes them out, fully coalesced.
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(tO + 32 * c, o);
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            pk[i] = pack_bf16x2(__uint_as_float(o[2 * i]) * inv, __uint_as_float(o[2 * i + 1]) * inv);
#pragma unroll
          for (int i = 0; i < 4; ++i)
            st_shared_v4(p_row + (c >> 1) * C::kPanelBytes + (((uint32_t)((c & 1) * 4 + i) ^ p_sw) << 4), pk[4 * i],
                         pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == 0) {
          const int y = (X ? w.qB_row0 : w.qA_row0) + 32 * wq;
          if (BAT_DCHECK(p.status, y >= 0 && y + 32 <= (p.T_suf - p.chk_shrink) && w.head >= 0 && w.head < p.H, kChkOutBulk, y)) {
#pragma unroll
            for (int pn = 0; pn < C::kPanels; ++pn)
              tma_store_2d(&p.tm_o, sm.p + X * C::kPTileBytes + pn * C::kPanelBytes + wq * 32 * 128, w.head * D + pn * 64,
                           y);
          }
          bulk_commit();
        }
        o_pending = true;
        BAT_TRACE_EV(3 + X, tn, 14, X, s_seen);
        if (p.lse && BAT_DCHECK(p.status, qrow >= 0 && qrow < (p.T_suf - p.chk_shrink) && w.head >= 0 && w.head < p.H, kChkLse, qrow))
          p.lse[(int64_t)w.head * p.T_suf + qrow] = lse2 * 0.69314718055994531f;
        o_stored = true;
      }
    }
    if (o_stored) {
    } else if (w.split_slot < 0) {
      __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(p.out) + ((int64_t)qrow * p.H + w.head) * D;
      const bool row_ok =
          !live || BAT_DCHECK(p.status, qrow >= 0 && qrow < (p.T_suf - p.chk_shrink) && w.head >= 0 && w.head < p.H, kChkOutRow, qrow);
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(tO + 32 * c, o);
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          pk[i] = pack_bf16x2(__uint_as_float(o[2 * i]) * inv, __uint_as_float(o[2 * i + 1]) * inv);
        if (live && row_ok) {
          uint4* d4 = reinterpret_cast<uint4*>(dst + 32 * c);
#pragma unroll
          for (int i = 0; i < 4; ++i) d4[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
        }
      }
      BAT_TRACE_EV(3 + X, tn, 14, X, s_seen);
      if (live && row_ok && p.lse) p.lse[(int64_t)w.head * p.T_suf + qrow] = lse2 * 0.69314718055994531f;
    } else {
      const int64_t slot = w.split_slot + X;
      float* dst = p.part_o + (slot * kTileM + row) * D;
      const bool part_ok = !live || BAT_DCHECK(p.status, slot >= 0 && slot < p.n_slots, kChkPartial, slot);
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(tO + 32 * c, o);
        if (live && part_ok) {
          float4* d4 = reinterpret_cast<float4*>(dst + 32 * c);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            d4[i] = make_float4(__uint_as_float(o[4 * i]) * inv, __uint_as_float(o[4 * i + 1]) * inv,
                                __uint_as_float(o[4 * i + 2]) * inv, __uint_as_float(o[4 * i + 3]) * inv);
        }
      }
      if (live && part_ok) p.part_lse[slot * kTileM + row] = lse2;
    }
  }
  BAT_PHASE_FLUSH();
  {
    // Bulk stores must be complete (and done reading shared memory) before the CTA exits.
    if (o_pending && lane == 0) bulk_wait_all();
    __syncwarp();
  }
}

template <int D>
__global__ void __launch_bounds__(kTcThreads, 1) bat_attn_tc_kernel(const __grid_constant__ TcParams p) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Smem<D> sm;
  sm.q = base;
  sm.p = base + 2 * C::kTileBytes;
  sm.kv = sm.p + C::kPBufs * C::kPTileBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm.kv + C::kStages * C::kTileBytes);
  sm.kv_full = bars;
  sm.kv_empty = bars + C::kStages;
  sm.q_full = sm.kv_empty + C::kStages;
  sm.q_empty = sm.q_full + 2;
  sm.s_full = sm.q_empty + 2;
  sm.s_free = sm.s_full + 2;
  sm.p_full = sm.s_free + 2;
  sm.pv_done = sm.p_full + 4;
  sm.drain = sm.pv_done + 4;
  sm.v_zeroed = sm.drain + 2;
  sm.itq_full = sm.v_zeroed + C::kStages;
  sm.itq_empty = sm.itq_full + kItemQ;
  sm.itq = reinterpret_cast<volatile int*>(sm.itq_empty + kItemQ);
  sm.tmem_slot = reinterpret_cast<uint32_t*>(const_cast<int*>(sm.itq) + kItemQ);
  sm.abort_flag = reinterpret_cast<volatile int*>(sm.tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(sm.kv_full + s, 1);
      mbar_init(sm.kv_empty + s, 2);   // one arrival per MMA issuer
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(sm.q_full + x, 1);
      mbar_init(sm.q_empty + x, 1);
      mbar_init(sm.s_full + x, 1);
      mbar_init(sm.s_free + x, 128);
      mbar_init(sm.p_full + 2 * x, 128);
      mbar_init(sm.p_full + 2 * x + 1, 128);
      mbar_init(sm.pv_done + 2 * x, 1);
      mbar_init(sm.pv_done + 2 * x + 1, 1);
    }
    mbar_init(sm.drain, 1);
    mbar_init(sm.drain + 1, 1);
    for (int s = 0; s < C::kStages; ++s) mbar_init(sm.v_zeroed + s, 1);
    for (int i = 0; i < kItemQ; ++i) {
      mbar_init(sm.itq_full + i, 1);
      mbar_init(sm.itq_empty + i, C::kItemConsumers);
    }
    *sm.abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 8 && (threadIdx.x & 31) == 0) {
    prefetch_tmap(&p.tm_q);
    prefetch_tmap(&p.tm_ks);
    prefetch_tmap(&p.tm_vs);
    prefetch_tmap(&p.tm_kc);
    prefetch_tmap(&p.tm_vc);
    prefetch_tmap(&p.tm_o);
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

  // Register split: the control warpgroup (producers, MMA issuers, idle warp) gives up
  // registers to the two softmax warpgroups.  384 threads x 168 at launch = 64512 =
  // 128 x 104 + 256 x 200.
  if (warp >= 8) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 104;" ::: "memory");
    if (warp == 8) producer_role<D>(p, sm, ctl);
    else if (warp == 9 || warp == 10) mma_role<D>(p, sm, ctl, tmem, warp - 9);
    else if constexpr (C::kTwoRings) vproducer_role<D>(p, sm, ctl);
    else qproducer_role<D>(p, sm, ctl);
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 200;" ::: "memory");
    softmax_role<D>(p, sm, ctl, tmem, warp >> 2);
  }

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
    cudaError_t e = cudaFuncSetAttribute(bat_attn_tc_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)Cfg<128>::kSmemBytes);
    if (e != cudaSuccess) return e;
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

#ifdef BAT_TRACE
extern "C" int bat_debug_set_trace(void* buf) {
  return (int)cudaMemcpyToSymbol(g_trace, &buf, sizeof(buf));
}
#elif defined(BAT_PHASE)
extern "C" int bat_debug_set_phase(void* buf) {
  return (int)cudaMemcpyToSymbol(g_phase, &buf, sizeof(buf));
}
#endif

cudaError_t device_status_word(uint32_t** out) {
  return cudaGetSymbolAddress(reinterpret_cast<void**>(out), g_status_word);
}

}  // namespace bat
