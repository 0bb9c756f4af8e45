// C ABI of libbat.so (declared in include/bat.h): argument checks, plan ownership,
// tensor-map encoding and kernel dispatch.  No computation of the operation happens here;
// every step of the forward runs in the library's kernels.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <vector>
#include <mutex>
#include <string>

#include "bat.h"
#include "bat_internal.h"
#include "bat_kernels.h"

struct bat_plan {
  bat::PlanResult host;
  bat::WorkItem* d_items = nullptr;
  bat::MergeJob* d_merges = nullptr;
  int32_t* d_counter = nullptr;   // work-item counter of the attention kernel
  int32_t R = 0, P = 0, H = 0, d = 0;
  bat_dtype dt = BAT_BF16;
  int64_t T_suf = 0, T_cache = 0;
  int64_t workspace_bytes = 0;
  int32_t num_sms = 148;
  int device = -1;
  bool on_device = false;
};

namespace {

thread_local std::string g_err;
std::atomic<uint64_t> g_wait_ns{2000000000ull};
constexpr uint64_t kDefaultWaitNs = 2000000000ull;

bat_status fail(bat_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_err = buf;
  return s;
}

bat_status cuda_fail(cudaError_t e, const char* what) {
  return fail(BAT_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool supported(bat_dtype dt, int32_t d) {
  if (dt == BAT_BF16) return d == 64 || d == 128;
  if (dt == BAT_FP32) return d == 32 || d == 64 || d == 128;
  return false;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static std::once_flag once;
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// 2-D map over a bf16 [T, H*d] row-major tensor: box 64 columns (128 bytes) x box_rows rows,
// 128-byte swizzle, zero fill outside the tensor.
bat_status encode_map(CUtensorMap* m, const void* base, int64_t T, int32_t H, int32_t d, const char* name,
                      uint32_t box_rows = bat::kTileN) {
  auto fn = encode_fn();
  if (!fn) return fail(BAT_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  cuuint64_t dims[2] = {(cuuint64_t)H * d, (cuuint64_t)(T > 0 ? T : 1)};
  cuuint64_t strides[1] = {(cuuint64_t)H * d * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(BAT_ERR_CUDA, "cuTensorMapEncodeTiled(%s) failed with CUresult %d", name, (int)r);
  return BAT_OK;
}

// Debug builds only: BAT_DEBUG_SHRINK_BOUNDS=n makes the device-side checks treat every tensor
// as n rows shorter than it is, so a valid run trips them on its last rows while every access
// the kernels still make stays inside the real tensors (a negative control of the checks).
int32_t debug_shrink() {
#ifdef BAT_DEBUG
  const char* e = getenv("BAT_DEBUG_SHRINK_BOUNDS");
  return e ? atoi(e) : 0;
#else
  return 0;
#endif
}

}  // namespace

namespace bat {
// Sets this thread's bat_last_error() message (for entry points defined in other files).
void set_last_error(const char* msg) { g_err = msg ? msg : ""; }
// The spin-wait limit set by bat_set_wait_timeout_ns (for kernels launched from other files).
uint64_t wait_limit_ns() { return g_wait_ns.load(); }
}  // namespace bat

extern "C" {

const char* bat_last_error(void) { return g_err.c_str(); }

int32_t bat_version(void) { return (1 << 16) | 1; }

int32_t bat_debug_checks(void) {
#ifdef BAT_DEBUG
  return 1;
#else
  return 0;
#endif
}

bat_status bat_set_wait_timeout_ns(uint64_t ns) {
  g_wait_ns.store(ns ? ns : kDefaultWaitNs);
  return BAT_OK;
}

bat_status bat_prefix_kv_build(const void* k_src, const void* v_src, const int64_t* src_offsets,
                               int32_t num_prefixes, const int64_t* dst_offsets, int32_t H, int32_t d,
                               bat_dtype dt, void* k_cache, void* v_cache, void* stream) {
  g_err.clear();
  if (num_prefixes < 0) return fail(BAT_ERR_INVALID_ARG, "num_prefixes=%d < 0", num_prefixes);
  if (num_prefixes == 0) return BAT_OK;
  if (!src_offsets || !dst_offsets) return fail(BAT_ERR_INVALID_ARG, "src_offsets and dst_offsets must be non-null");
  if (H <= 0 || d <= 0) return fail(BAT_ERR_INVALID_ARG, "H=%d and d=%d must be > 0", H, d);
  if (dt != BAT_BF16 && dt != BAT_FP32) return fail(BAT_ERR_INVALID_ARG, "unknown dtype %d", (int)dt);
  const int64_t row_bytes = (int64_t)H * d * (dt == BAT_BF16 ? 2 : 4);
  if (row_bytes % 16) return fail(BAT_ERR_INVALID_ARG, "row bytes H*d*elt=%lld not a multiple of 16", (long long)row_bytes);
  if (src_offsets[0] < 0) return fail(BAT_ERR_INVALID_ARG, "src_offsets[0] < 0");
  int64_t total = 0;
  for (int32_t i = 0; i < num_prefixes; ++i) {
    if (src_offsets[i + 1] < src_offsets[i])
      return fail(BAT_ERR_INVALID_ARG, "src_offsets not monotone at %d", i);
    if (dst_offsets[i] < 0) return fail(BAT_ERR_INVALID_ARG, "dst_offsets[%d] < 0", i);
    total += src_offsets[i + 1] - src_offsets[i];
  }
  if (total == 0) return BAT_OK;
  if (!k_src || !v_src || !k_cache || !v_cache)
    return fail(BAT_ERR_INVALID_ARG, "k_src, v_src, k_cache, v_cache must be non-null");
  if (!aligned16(k_src) || !aligned16(v_src) || !aligned16(k_cache) || !aligned16(v_cache))
    return fail(BAT_ERR_INVALID_ARG, "device pointers must be 16-byte aligned");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  bat::PackBatch b;
  memset(&b, 0, sizeof(b));
  int64_t max_bytes = 0;
  for (int32_t i = 0; i < num_prefixes; ++i) {
    const int64_t rows = src_offsets[i + 1] - src_offsets[i];
    if (rows == 0) continue;
    b.src_byte[b.n] = src_offsets[i] * row_bytes;
    b.dst_byte[b.n] = dst_offsets[i] * row_bytes;
    b.bytes[b.n] = rows * row_bytes;
    max_bytes = std::max(max_bytes, b.bytes[b.n]);
    if (++b.n == bat::kPackBatch) {
      cudaError_t e = bat::launch_pack(k_src, v_src, k_cache, v_cache, b, max_bytes, s);
      if (e != cudaSuccess) return cuda_fail(e, "pack kernel launch");
      b.n = 0;
      max_bytes = 0;
    }
  }
  if (b.n) {
    cudaError_t e = bat::launch_pack(k_src, v_src, k_cache, v_cache, b, max_bytes, s);
    if (e != cudaSuccess) return cuda_fail(e, "pack kernel launch");
  }
  return BAT_OK;
}

bat_status bat_plan_create(const int32_t* req_prefix, const int64_t* suffix_offsets, const int64_t* prefix_offsets,
                           int32_t R, int32_t P, int32_t H, int32_t d, bat_dtype dt, const bat_plan_options* opts,
                           void* stream, bat_plan** out) {
  g_err.clear();
  if (!out) return fail(BAT_ERR_INVALID_ARG, "out must be non-null");
  *out = nullptr;
  if (!supported(dt, d))
    return fail(BAT_ERR_UNSUPPORTED, "dtype %d with d=%d is not supported (bf16: d in {64,128}; fp32: d in {32,64,128})",
                (int)dt, d);
  bat_plan_options o;
  memset(&o, 0, sizeof(o));
  if (opts) o = *opts;
  for (int i = 0; i < 4; ++i)
    if (o.reserved[i]) return fail(BAT_ERR_INVALID_ARG, "bat_plan_options.reserved must be zero");
  if (o.split_mode < 0 || o.split_mode > 2) return fail(BAT_ERR_INVALID_ARG, "split_mode %d not in {0,1,2}", o.split_mode);
  if (o.split_chunk_tiles < 0) return fail(BAT_ERR_INVALID_ARG, "split_chunk_tiles < 0");

  bat_plan* plan = new (std::nothrow) bat_plan();
  if (!plan) return fail(BAT_ERR_OOM, "out of host memory");
  plan->R = R;
  plan->P = P;
  plan->H = H;
  plan->d = d;
  plan->dt = dt;
  plan->T_suf = (R > 0 && suffix_offsets) ? suffix_offsets[R] : 0;
  plan->T_cache = (P > 0 && prefix_offsets) ? prefix_offsets[P] : 0;
  int num_sms = o.num_sms;
  if (num_sms <= 0) {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) == cudaSuccess &&
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && n > 0)
      num_sms = n;
    else
      num_sms = 148;
    cudaGetLastError();   // a host-only plan on a machine without a GPU is fine
  }
  plan->num_sms = num_sms;
  bat::PlanOptions po{o.split_mode, o.split_chunk_tiles, num_sms};
  char err[400] = {0};
  if (bat::build_plan(req_prefix, suffix_offsets, prefix_offsets, R, P, H, po, &plan->host, err, sizeof(err))) {
    delete plan;
    return fail(BAT_ERR_INVALID_ARG, "%s", err);
  }
  const int64_t elt = 4;
  plan->workspace_bytes = plan->host.n_slots * (int64_t)bat::kTileM * (d * elt + 4);
  if (!o.host_only) {
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaGetDevice(&plan->device);
    if (e != cudaSuccess) {
      bat::free_plan_result(&plan->host);
      delete plan;
      return cuda_fail(e, "cudaGetDevice");
    }
    const size_t ib = plan->host.n_items * sizeof(bat::WorkItem), mb = plan->host.n_merges * sizeof(bat::MergeJob);
    if (ib) e = cudaMalloc(&plan->d_items, ib);
    if (e == cudaSuccess && mb) e = cudaMalloc(&plan->d_merges, mb);
    if (e == cudaSuccess) e = cudaMalloc(&plan->d_counter, 16);
    if (e == cudaSuccess && ib) e = cudaMemcpyAsync(plan->d_items, plan->host.items, ib, cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess && mb) e = cudaMemcpyAsync(plan->d_merges, plan->host.merges, mb, cudaMemcpyHostToDevice, s);
    if (e != cudaSuccess) {
      cudaFree(plan->d_items);
      cudaFree(plan->d_merges);
      cudaFree(plan->d_counter);
      bat::free_plan_result(&plan->host);
      delete plan;
      return e == cudaErrorMemoryAllocation ? fail(BAT_ERR_OOM, "device allocation of the work list failed")
                                            : cuda_fail(e, "work list upload");
    }
    plan->on_device = true;
  }
  *out = plan;
  return BAT_OK;
}

bat_status bat_plan_create_prefix_side(const int64_t* src_offsets, int32_t num_prefixes, int32_t H, int32_t d,
                                       bat_dtype dt, const bat_plan_options* opts, void* stream, bat_plan** out) {
  g_err.clear();
  if (num_prefixes < 0) return fail(BAT_ERR_INVALID_ARG, "num_prefixes=%d < 0", num_prefixes);
  if (num_prefixes > 0 && !src_offsets) return fail(BAT_ERR_INVALID_ARG, "src_offsets must be non-null");
  // Every prefix becomes a request with no cached prefix whose own tokens are the prefix's.
  std::vector<int32_t> req_prefix((size_t)num_prefixes, -1);
  const int64_t no_cache[1] = {0};
  const int64_t empty_so[1] = {0};
  return bat_plan_create(num_prefixes ? req_prefix.data() : nullptr, num_prefixes ? src_offsets : empty_so,
                         no_cache, num_prefixes, 0, H, d, dt, opts, stream, out);
}

bat_status bat_plan_destroy(bat_plan* plan) {
  g_err.clear();
  if (!plan) return BAT_OK;
  bat_status st = BAT_OK;
  if (plan->on_device) {
    int cur = -1;
    cudaGetDevice(&cur);
    if (cur != plan->device) cudaSetDevice(plan->device);
    cudaError_t e1 = cudaFree(plan->d_items), e2 = cudaFree(plan->d_merges);
    cudaFree(plan->d_counter);
    if (cur >= 0 && cur != plan->device) cudaSetDevice(cur);
    if (e1 != cudaSuccess || e2 != cudaSuccess) st = cuda_fail(e1 != cudaSuccess ? e1 : e2, "cudaFree of the work list");
  }
  bat::free_plan_result(&plan->host);
  delete plan;
  return st;
}

bat_status bat_plan_info(const bat_plan* plan, bat_plan_info_t* info) {
  g_err.clear();
  if (!plan || !info) return fail(BAT_ERR_INVALID_ARG, "plan and info must be non-null");
  memset(info, 0, sizeof(*info));
  info->n_items = plan->host.n_items;
  info->n_merges = plan->host.n_merges;
  info->n_slots = plan->host.n_slots;
  info->workspace_bytes = plan->workspace_bytes;
  info->total_cost = plan->host.total_cost;
  info->T_suf = plan->T_suf;
  info->T_cache = plan->T_cache;
  info->R = plan->R;
  info->P = plan->P;
  info->H = plan->H;
  info->d = plan->d;
  info->dtype = (int32_t)plan->dt;
  info->on_device = plan->on_device ? 1 : 0;
  return BAT_OK;
}

size_t bat_workspace_bytes(const bat_plan* plan) { return plan ? (size_t)plan->workspace_bytes : 0; }

bat_status bat_plan_items(const bat_plan* plan, void* dst, size_t dst_bytes) {
  g_err.clear();
  if (!plan || (!dst && plan->host.n_items)) return fail(BAT_ERR_INVALID_ARG, "plan and dst must be non-null");
  const size_t need = plan->host.n_items * sizeof(bat::WorkItem);
  if (dst_bytes < need) return fail(BAT_ERR_INVALID_ARG, "dst has %zu bytes, need %zu", dst_bytes, need);
  if (need) memcpy(dst, plan->host.items, need);
  return BAT_OK;
}

bat_status bat_plan_merges(const bat_plan* plan, void* dst, size_t dst_bytes) {
  g_err.clear();
  if (!plan || (!dst && plan->host.n_merges)) return fail(BAT_ERR_INVALID_ARG, "plan and dst must be non-null");
  const size_t need = plan->host.n_merges * sizeof(bat::MergeJob);
  if (dst_bytes < need) return fail(BAT_ERR_INVALID_ARG, "dst has %zu bytes, need %zu", dst_bytes, need);
  if (need) memcpy(dst, plan->host.merges, need);
  return BAT_OK;
}

bat_status bat_attention_forward(const bat_plan* plan, const void* q, const void* k_suf, const void* v_suf,
                                 const void* k_cache, const void* v_cache, float scale, bat_dtype dt, void* out,
                                 float* lse, void* workspace, size_t workspace_bytes, void* stream) {
  g_err.clear();
  if (!plan) return fail(BAT_ERR_INVALID_ARG, "plan must be non-null");
  if (!plan->on_device) return fail(BAT_ERR_INVALID_ARG, "the plan was built host-only and cannot run");
  if (dt != plan->dt) return fail(BAT_ERR_INVALID_ARG, "dtype %d differs from the plan's %d", (int)dt, (int)plan->dt);
  if (plan->host.n_items == 0) return BAT_OK;
  if (!q || !k_suf || !v_suf || !out) return fail(BAT_ERR_INVALID_ARG, "q, k_suf, v_suf and out must be non-null");
  if (plan->T_cache > 0 && (!k_cache || !v_cache))
    return fail(BAT_ERR_INVALID_ARG, "k_cache and v_cache must be non-null when the cache has %lld rows",
                (long long)plan->T_cache);
  if (!aligned16(q) || !aligned16(k_suf) || !aligned16(v_suf) || !aligned16(out) ||
      (k_cache && !aligned16(k_cache)) || (v_cache && !aligned16(v_cache)))
    return fail(BAT_ERR_INVALID_ARG, "device pointers must be 16-byte aligned");
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return fail(BAT_ERR_INVALID_ARG, "lse must be 4-byte aligned");
  if (plan->workspace_bytes > 0) {
    if (!workspace || (int64_t)workspace_bytes < plan->workspace_bytes)
      return fail(BAT_ERR_INVALID_ARG, "workspace needs %lld bytes, got %zu", (long long)plan->workspace_bytes,
                  workspace_bytes);
    if (!aligned16(workspace)) return fail(BAT_ERR_INVALID_ARG, "workspace must be 16-byte aligned");
  }
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev != plan->device)
    return fail(BAT_ERR_INVALID_ARG, "the current device %d is not the plan's device %d", dev, plan->device);
  const float sc = scale > 0.f ? scale : 1.0f / std::sqrt((float)plan->d);
  if (!std::isfinite(sc)) return fail(BAT_ERR_INVALID_ARG, "scale must be finite");
  uint32_t* status = nullptr;
  e = bat::device_status_word(&status);
  if (e != cudaSuccess) return cuda_fail(e, "device status word");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  float* part_o = static_cast<float*>(workspace);
  float* part_lse = part_o ? part_o + plan->host.n_slots * (int64_t)bat::kTileM * plan->d : nullptr;

  if (dt == BAT_BF16) {
    bat::TcParams p;
    memset(&p, 0, sizeof(p));
    bat_status st;
    if ((st = encode_map(&p.tm_q, q, plan->T_suf, plan->H, plan->d, "q")) != BAT_OK) return st;
    if ((st = encode_map(&p.tm_ks, k_suf, plan->T_suf, plan->H, plan->d, "k_suf")) != BAT_OK) return st;
    if ((st = encode_map(&p.tm_vs, v_suf, plan->T_suf, plan->H, plan->d, "v_suf")) != BAT_OK) return st;
    const bool has_cache = plan->T_cache > 0;
    if ((st = encode_map(&p.tm_kc, has_cache ? k_cache : k_suf, has_cache ? plan->T_cache : plan->T_suf, plan->H,
                         plan->d, "k_cache")) != BAT_OK)
      return st;
    if ((st = encode_map(&p.tm_vc, has_cache ? v_cache : v_suf, has_cache ? plan->T_cache : plan->T_suf, plan->H,
                         plan->d, "v_cache")) != BAT_OK)
      return st;
    // The output map stores one warp's 32 rows at a time (rows of a partial query tile that
    // belong to another request are never covered: such warps store row by row instead).
    if ((st = encode_map(&p.tm_o, out, plan->T_suf, plan->H, plan->d, "out", 32)) != BAT_OK) return st;
    p.items = plan->d_items;
    p.n_items = plan->host.n_items;
    p.out = out;
    p.lse = lse;
    p.part_o = part_o;
    p.part_lse = part_lse;
    p.T_suf = (int32_t)plan->T_suf;
    p.H = plan->H;
    p.scale_log2 = sc * 1.4426950408889634f;
    p.status = status;
    p.wait_ns = g_wait_ns.load();
    p.item_counter = plan->d_counter;
    p.T_cache = (int32_t)(has_cache ? plan->T_cache : plan->T_suf);
    p.n_slots = (int32_t)plan->host.n_slots;
    p.chk_shrink = debug_shrink();
    e = cudaMemsetAsync(plan->d_counter, 0, sizeof(int32_t), s);
    if (e != cudaSuccess) return cuda_fail(e, "resetting the work-item counter");
    const int grid = (int)std::min<int64_t>(plan->host.n_items, plan->num_sms);
    e = bat::launch_attn_tc(plan->d, p, grid, s);
    if (e != cudaSuccess) return cuda_fail(e, "attention kernel launch");
  } else {
    bat::SimtParams p;
    memset(&p, 0, sizeof(p));
    p.items = plan->d_items;
    p.n_items = plan->host.n_items;
    p.q = static_cast<const float*>(q);
    p.ks = static_cast<const float*>(k_suf);
    p.vs = static_cast<const float*>(v_suf);
    p.kc = static_cast<const float*>(k_cache);
    p.vc = static_cast<const float*>(v_cache);
    p.out = static_cast<float*>(out);
    p.lse = lse;
    p.part_o = part_o;
    p.part_lse = part_lse;
    p.T_suf = (int32_t)plan->T_suf;
    p.H = plan->H;
    p.scale = sc;
    p.T_cache = (int32_t)plan->T_cache;
    p.n_slots = (int32_t)plan->host.n_slots;
    p.status = status;
    p.chk_shrink = debug_shrink();
    e = bat::launch_attn_simt(plan->d, p, s);
    if (e != cudaSuccess) return cuda_fail(e, "fp32 attention kernel launch");
  }
  if (plan->host.n_merges > 0) {
    bat::MergeParams m;
    m.jobs = plan->d_merges;
    m.n_jobs = plan->host.n_merges;
    m.part_o = part_o;
    m.part_lse = part_lse;
    m.out = out;
    m.lse = lse;
    m.T_suf = (int32_t)plan->T_suf;
    m.H = plan->H;
    m.n_slots = (int32_t)plan->host.n_slots;
    m.status = status;
    m.chk_shrink = debug_shrink();
    e = bat::launch_merge(plan->d, dt == BAT_BF16, m, s);
    if (e != cudaSuccess) return cuda_fail(e, "merge kernel launch");
  }
  return BAT_OK;
}

bat_status bat_get_device_status(void* stream) {
  g_err.clear();
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  uint32_t* word = nullptr;
  e = bat::device_status_word(&word);
  if (e != cudaSuccess) return cuda_fail(e, "device status word");
  uint32_t v[3] = {0, 0, 0};
  e = cudaMemcpy(v, word, sizeof(v), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "reading the device status word");
  if (v[0]) {
    e = cudaMemset(word, 0, sizeof(v));
    if (e != cudaSuccess) return cuda_fail(e, "clearing the device status word");
    if (v[0] & 2u)
      return fail(BAT_ERR_DEVICE_CHECK,
                  "a device-side bounds check failed (check %u, value %u; status 0x%x); the access was skipped",
                  v[1], v[2], v[0]);
    return fail(BAT_ERR_TIMEOUT, "a kernel abandoned a bounded wait (status 0x%x); its outputs are incomplete", v[0]);
  }
  return BAT_OK;
}

}  // extern "C"
