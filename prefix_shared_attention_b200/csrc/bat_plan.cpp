// Host grouping pass: bucket requests by the cached prefix they read and emit the work list.
//
// Bat lead page, section "Why it works": a hot item's cached K/V serves the many users who
// see it, and a user's cached K/V serves all of that user's requests.  The pass makes that
// sharing explicit for the kernel: the query tiles of requests with the same prefix are
// paired into work items that stream the prefix K/V tiles once for both tiles, and the
// items of one prefix are emitted next to each other so concurrently running CTAs hit the
// same prefix tiles in L2.
#include <algorithm>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <limits>
#include <vector>

#include "bat_internal.h"

namespace bat {
namespace {

inline int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

struct QTile {
  int32_t req, row0, rows;
};

int fail(char* err, size_t n, const char* fmt, long long a = 0, long long b = 0, long long c = 0) {
  if (err && n) snprintf(err, n, fmt, a, b, c);
  return 1;
}

int64_t item_cost(const WorkItem& w) {
  int64_t npre = cdiv(w.pre_len, kTileN);
  if (w.n_q == 1) return npre + cdiv(w.sA_len, kTileN);
  if (w.shared) return 2 * (npre + cdiv(w.sA_len, kTileN));
  return 2 * npre + cdiv(w.sA_len, kTileN) + cdiv(w.sB_len, kTileN);
}

// Key tiles a shared-stream item walks: the prefix tiles, then the suffix tiles.
int64_t stream_tiles(const WorkItem& w) {
  return cdiv(w.pre_len, kTileN) + cdiv(w.sA_len, kTileN);
}

}  // namespace

void free_plan_result(PlanResult* r) {
  if (!r) return;
  free(r->items);
  free(r->merges);
  *r = PlanResult();
}

int build_plan(const int32_t* req_prefix, const int64_t* suffix_offsets,
               const int64_t* prefix_offsets, int32_t R, int32_t P, int32_t H,
               const PlanOptions& opt, PlanResult* out, char* err, size_t err_len) {
  const int64_t kMaxRows = std::numeric_limits<int32_t>::max() - 2 * kTileN;
  *out = PlanResult();
  if (R < 0 || P < 0) return fail(err, err_len, "R=%lld and P=%lld must be >= 0", R, P);
  if (H <= 0) return fail(err, err_len, "H=%lld must be > 0", H);
  if (R > 0 && (!req_prefix || !suffix_offsets))
    return fail(err, err_len, "req_prefix and suffix_offsets must be non-null when R=%lld > 0", R);
  if (P > 0 && !prefix_offsets) return fail(err, err_len, "prefix_offsets must be non-null when P=%lld > 0", P);
  if (R > 0) {
    if (suffix_offsets[0] < 0) return fail(err, err_len, "suffix_offsets[0]=%lld is negative", suffix_offsets[0]);
    for (int32_t r = 0; r < R; ++r) {
      if (suffix_offsets[r + 1] < suffix_offsets[r])
        return fail(err, err_len, "suffix_offsets not monotone at request %lld (%lld > %lld)", r,
                    suffix_offsets[r], suffix_offsets[r + 1]);
      if (req_prefix[r] < -1 || req_prefix[r] >= P)
        return fail(err, err_len, "req_prefix[%lld]=%lld out of range [-1, %lld)", r, req_prefix[r], P);
    }
    if (suffix_offsets[R] > kMaxRows)
      return fail(err, err_len, "suffix rows %lld exceed the int32 row limit %lld", suffix_offsets[R], kMaxRows);
  }
  if (P > 0) {
    if (prefix_offsets[0] < 0) return fail(err, err_len, "prefix_offsets[0]=%lld is negative", prefix_offsets[0]);
    for (int32_t p = 0; p < P; ++p)
      if (prefix_offsets[p + 1] < prefix_offsets[p])
        return fail(err, err_len, "prefix_offsets not monotone at prefix %lld (%lld > %lld)", p,
                    prefix_offsets[p], prefix_offsets[p + 1]);
    if (prefix_offsets[P] > kMaxRows)
      return fail(err, err_len, "cache rows %lld exceed the int32 row limit %lld", prefix_offsets[P], kMaxRows);
  }
  const int num_sms = opt.num_sms > 0 ? opt.num_sms : 148;

  // Counting sort of the requests by prefix id; bucket 0 holds the requests with none.
  std::vector<int64_t> start(P + 2, 0);
  for (int32_t r = 0; r < R; ++r) start[req_prefix[r] + 2]++;
  for (int32_t b = 1; b < P + 2; ++b) start[b] += start[b - 1];
  std::vector<int32_t> by_prefix(R);
  {
    std::vector<int64_t> pos(start.begin(), start.end() - 1);
    for (int32_t r = 0; r < R; ++r) by_prefix[pos[req_prefix[r] + 1]++] = r;
  }

  // Items of every group, before they are replicated over heads.
  struct Group {
    int32_t prefix;
    std::vector<WorkItem> items;
    int64_t cost = 0;
  };
  std::vector<Group> groups;
  groups.reserve(P + 1);
  for (int32_t b = 0; b < P + 1; ++b) {
    const int32_t p = b - 1;
    Group g;
    g.prefix = p;
    const int32_t pre_row0 = p >= 0 ? (int32_t)prefix_offsets[p] : 0;
    const int32_t pre_len = p >= 0 ? (int32_t)(prefix_offsets[p + 1] - prefix_offsets[p]) : 0;
    std::vector<QTile> leftovers;
    auto base = [&](void) {
      WorkItem w;
      memset(&w, 0, sizeof(w));
      w.split_slot = -1;
      w.pre_row0 = pre_row0;
      w.pre_len = pre_len;
      w.group = p;
      return w;
    };
    for (int64_t i = start[b]; i < start[b + 1]; ++i) {
      const int32_t r = by_prefix[i];
      const int32_t s0 = (int32_t)suffix_offsets[r];
      const int32_t Ls = (int32_t)(suffix_offsets[r + 1] - suffix_offsets[r]);
      if (Ls == 0) continue;
      const int32_t nt = (int32_t)cdiv(Ls, kTileM);
      // Two query tiles of one request share every key tile: prefix and suffix.
      for (int32_t k = 0; k + 1 < nt; k += 2) {
        WorkItem w = base();
        w.n_q = 2;
        w.shared = 1;
        w.qA_row0 = s0 + k * kTileM;
        w.qA_rows = std::min(kTileM, Ls - k * kTileM);
        w.qB_row0 = s0 + (k + 1) * kTileM;
        w.qB_rows = std::min(kTileM, Ls - (k + 1) * kTileM);
        w.sA_row0 = w.sB_row0 = s0;
        w.sA_len = w.sB_len = Ls;
        g.items.push_back(w);
      }
      if (nt & 1) leftovers.push_back({r, s0 + (nt - 1) * kTileM, Ls - (nt - 1) * kTileM});
    }
    // Odd tiles of different requests in the group: they share the prefix tiles only.
    size_t i = 0;
    for (; i + 1 < leftovers.size(); i += 2) {
      const QTile &a = leftovers[i], &c = leftovers[i + 1];
      WorkItem w = base();
      w.n_q = 2;
      w.shared = 0;
      w.qA_row0 = a.row0;
      w.qA_rows = a.rows;
      w.sA_row0 = (int32_t)suffix_offsets[a.req];
      w.sA_len = (int32_t)(suffix_offsets[a.req + 1] - suffix_offsets[a.req]);
      w.qB_row0 = c.row0;
      w.qB_rows = c.rows;
      w.sB_row0 = (int32_t)suffix_offsets[c.req];
      w.sB_len = (int32_t)(suffix_offsets[c.req + 1] - suffix_offsets[c.req]);
      g.items.push_back(w);
    }
    if (i < leftovers.size()) {
      const QTile& a = leftovers[i];
      WorkItem w = base();
      w.n_q = 1;
      w.shared = 1;
      w.qA_row0 = a.row0;
      w.qA_rows = a.rows;
      w.sA_row0 = w.sB_row0 = (int32_t)suffix_offsets[a.req];
      w.sA_len = w.sB_len = (int32_t)(suffix_offsets[a.req + 1] - suffix_offsets[a.req]);
      g.items.push_back(w);
    }
    for (auto& w : g.items) {
      w.cost = (int32_t)item_cost(w);
      g.cost += w.cost;
    }
    if (!g.items.empty()) groups.push_back(std::move(g));
  }

  int64_t total_cost = 0;
  for (auto& g : groups) total_cost += g.cost * H;

  // Split pass: a shared-stream item far heavier than one SM's fair share is cut into
  // chunks of consecutive key tiles whose partials are merged by log-sum-exp afterwards.
  struct Chunking {
    int32_t n_chunks = 1;
  };
  const int64_t fair = std::max<int64_t>(1, total_cost / num_sms);
  auto chunks_for = [&](const WorkItem& w) -> int32_t {
    if (opt.split_mode == 1) return 1;
    if (!(w.n_q == 1 || w.shared)) return 1;
    const int64_t nkv = stream_tiles(w);
    if (nkv < 2) return 1;
    int64_t n;
    if (opt.split_mode == 2) {
      const int64_t per = opt.split_chunk_tiles > 0 ? opt.split_chunk_tiles : 2;
      n = std::max<int64_t>(2, cdiv(nkv, per));
    } else {
      if (w.cost * 2 <= fair) return 1;
      const int64_t per = opt.split_chunk_tiles > 0 ? opt.split_chunk_tiles
                                                    : std::max<int64_t>(2, fair / (4 * w.n_q));
      n = cdiv(nkv, per);
    }
    return (int32_t)std::min<int64_t>(n, nkv);
  };

  // Order: heaviest group first; within a group, every head in turn, items heaviest first.
  std::stable_sort(groups.begin(), groups.end(),
                   [](const Group& a, const Group& b) { return a.cost > b.cost; });
  // Chunk counts per group item (the same for every head), and the exact output sizes.
  std::vector<std::vector<int32_t>> nchs(groups.size());
  int64_t n_items_total = 0, n_merges_total = 0;
  for (size_t gi = 0; gi < groups.size(); ++gi) {
    auto& g = groups[gi];
    std::stable_sort(g.items.begin(), g.items.end(),
                     [](const WorkItem& a, const WorkItem& b) { return a.cost > b.cost; });
    nchs[gi].resize(g.items.size());
    for (size_t i = 0; i < g.items.size(); ++i) {
      const int32_t nch = chunks_for(g.items[i]);
      nchs[gi][i] = nch;
      n_items_total += (int64_t)nch * H;
      if (nch > 1) n_merges_total += (int64_t)g.items[i].n_q * H;
    }
  }
  // The work list is written straight into the result's buffers.
  if (n_items_total > 0) {
    out->items = (WorkItem*)malloc((size_t)n_items_total * sizeof(WorkItem));
    if (!out->items) return fail(err, err_len, "out of host memory for %lld work items", (long long)n_items_total);
  }
  if (n_merges_total > 0) {
    out->merges = (MergeJob*)malloc((size_t)n_merges_total * sizeof(MergeJob));
    if (!out->merges) {
      free_plan_result(out);
      return fail(err, err_len, "out of host memory for %lld merge jobs", (long long)n_merges_total);
    }
  }
  WorkItem* items = out->items;
  MergeJob* merges = out->merges;
  int64_t ni = 0, nm = 0;
  int64_t n_slots = 0;
  for (size_t gi = 0; gi < groups.size(); ++gi) {
    const auto& g = groups[gi];
    for (int32_t h = 0; h < H; ++h) {
      for (size_t ii = 0; ii < g.items.size(); ++ii) {
        const WorkItem& w0 = g.items[ii];
        const int32_t nch = nchs[gi][ii];
        if (nch <= 1) {
          WorkItem& w = items[ni++];
          w = w0;
          w.head = h;
          continue;
        }
        const int64_t npre = cdiv(w0.pre_len, kTileN);
        const int64_t nkv = stream_tiles(w0);
        const int64_t slot0 = n_slots;
        for (int32_t c = 0; c < nch; ++c) {
          const int64_t t0 = (nkv * c) / nch, t1 = (nkv * (c + 1)) / nch;   // key tiles [t0, t1)
          WorkItem w = w0;
          w.head = h;
          w.split_slot = (int32_t)(slot0 + (int64_t)c * w0.n_q);
          // Prefix part of the chunk.
          const int64_t p0 = std::min(t0, npre), p1 = std::min(t1, npre);
          w.pre_row0 = w0.pre_row0 + (int32_t)(p0 * kTileN);
          w.pre_len = p1 > p0 ? (int32_t)(std::min<int64_t>(p1 * kTileN, w0.pre_len) - p0 * kTileN) : 0;
          // Suffix part of the chunk.
          const int64_t s0 = std::max<int64_t>(t0 - npre, 0), s1 = std::max<int64_t>(t1 - npre, 0);
          w.sA_row0 = w0.sA_row0 + (int32_t)(s0 * kTileN);
          w.sA_len = s1 > s0 ? (int32_t)(std::min<int64_t>(s1 * kTileN, w0.sA_len) - s0 * kTileN) : 0;
          w.sB_row0 = w.sA_row0;
          w.sB_len = w.sA_len;
          w.cost = (int32_t)item_cost(w);
          items[ni++] = w;
        }
        n_slots += (int64_t)nch * w0.n_q;
        for (int32_t x = 0; x < w0.n_q; ++x) {
          MergeJob m;
          memset(&m, 0, sizeof(m));
          m.q_row0 = x == 0 ? w0.qA_row0 : w0.qB_row0;
          m.q_rows = x == 0 ? w0.qA_rows : w0.qB_rows;
          m.head = h;
          m.slot0 = (int32_t)(slot0 + x);
          m.n_chunks = nch;
          m.slot_stride = w0.n_q;
          merges[nm++] = m;
        }
      }
    }
  }
  if (n_slots > std::numeric_limits<int32_t>::max() / 2) {
    free_plan_result(out);
    return fail(err, err_len, "too many split slots (%lld)", n_slots);
  }
  if (ni != n_items_total || nm != n_merges_total) {
    free_plan_result(out);
    return fail(err, err_len, "internal: %lld work items and %lld merge jobs written, not the sizes counted",
                (long long)ni, (long long)nm);
  }
  out->n_items = ni;
  out->n_merges = nm;
  out->n_slots = n_slots;
  out->total_cost = total_cost;
  return 0;
}

}  // namespace bat
