// Internal definitions shared by the library's host code and kernels.
//
// The work list is the product of the host grouping pass: requests that read the same
// cached prefix are bucketed together, and each work item pairs up to two 128-row query
// tiles of one head that stream the same prefix K/V tiles (Bat lead page, section
// "Why it works": one cached computation serves every query that shares it).
#pragma once

#include <cstddef>
#include <cstdint>

namespace bat {

constexpr int kTileM = 128;   // query rows per Q tile (TMEM lanes)
constexpr int kTileN = 128;   // keys per K/V tile

// One unit of kernel work: head `head`, Q tile A (and optionally B), and the key ranges
// they attend over.  All row indices are absolute rows of the [T, H, d] tensors.
struct WorkItem {
  int32_t head;
  int32_t n_q;          // 1 or 2 query tiles
  int32_t shared;       // 1: tile B reads the same suffix keys as tile A (same request)
  int32_t split_slot;   // -1: write the output directly; else partial slot of tile A (B: +1)
  int32_t pre_row0;     // first cache row of this item's prefix keys
  int32_t pre_len;      // prefix keys in this item (0 = none)
  int32_t qA_row0, qA_rows, sA_row0, sA_len;   // tile A: query rows, suffix key range
  int32_t qB_row0, qB_rows, sB_row0, sB_len;   // tile B (unused when n_q == 1)
  int32_t cost;         // score tiles (128x128) computed by the item
  int32_t group;        // prefix id (-1: none); diagnostics only
};
static_assert(sizeof(WorkItem) == 64, "WorkItem is 64 bytes");

// Log-sum-exp merge of the partials that a split query tile produced.
struct MergeJob {
  int32_t q_row0, q_rows, head, slot0;
  int32_t n_chunks, slot_stride, pad0, pad1;
};
static_assert(sizeof(MergeJob) == 32, "MergeJob is 32 bytes");

struct PlanOptions {
  int32_t split_mode;         // 0 auto, 1 never, 2 always (every splittable item)
  int32_t split_chunk_tiles;  // 0 auto; else key tiles per chunk when splitting
  int32_t num_sms;            // SMs to balance over
};

struct PlanResult {
  WorkItem* items = nullptr;
  int64_t n_items = 0;
  MergeJob* merges = nullptr;
  int64_t n_merges = 0;
  int64_t n_slots = 0;
  int64_t total_cost = 0;
};

// Host grouping pass. Returns 0 on success, else writes a message into `err`.
int build_plan(const int32_t* req_prefix, const int64_t* suffix_offsets,
               const int64_t* prefix_offsets, int32_t R, int32_t P, int32_t H,
               const PlanOptions& opt, PlanResult* out, char* err, size_t err_len);
void free_plan_result(PlanResult* r);

}  // namespace bat
