// C ABI of the GBLA path (declared in include/bat.h): the work list of a batch of user
// histories, argument checks and the kernel launches.  No arithmetic of the layer happens
// here; it all runs in bat_gbla.cu's kernels.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <mutex>
#include <cstdio>
#include <cstring>
#include <new>
#include <vector>

#include "bat.h"
#include "bat_gbla_internal.h"
#include "bat_kernels.h"

namespace bat {
void set_last_error(const char* msg);
}

struct bat_gbla_plan {
  std::vector<bat::GblaChunk> chunks;
  std::vector<bat::GblaPair> pairs;
  bat::GblaChunk* d_chunks = nullptr;
  bat::GblaPair* d_pairs = nullptr;
  int32_t n_seqs = 0, H = 0, d = 0;
  int64_t T = 0;
  int64_t workspace_bytes = 0;
  int device = -1;
  bool on_device = false;
};

namespace {

bat_status gfail(bat_status s, const char* fmt, long long a = 0, long long b = 0) {
  char buf[300];
  snprintf(buf, sizeof(buf), fmt, a, b);
  bat::set_last_error(buf);
  return s;
}

bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

constexpr int64_t kPartFloats = 128 * 128 + 128;

int64_t align256(int64_t x) { return (x + 255) & ~int64_t(255); }

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

// 2-D map over a bf16 [T, H*128] tensor: box 64 columns x box_rows rows; zero fill outside it.
bool encode(CUtensorMap* m, const void* base, int64_t T, int32_t H, uint32_t box_rows, bool swizzle128) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)H * 128, (cuuint64_t)(T > 0 ? T : 1)};
  cuuint64_t strides[1] = {(cuuint64_t)H * 128 * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

extern "C" {

bat_status bat_gbla_plan_create(const int64_t* seq_offsets, int32_t n_seqs, int32_t H, int32_t d, int32_t num_sms,
                                int32_t host_only, void* stream, bat_gbla_plan** out) {
  bat::set_last_error("");
  if (!out) return gfail(BAT_ERR_INVALID_ARG, "out must be non-null");
  *out = nullptr;
  if (d != 128) return gfail(BAT_ERR_UNSUPPORTED, "GBLA runs at d = 128 only (got d=%lld)", d);
  if (H <= 0) return gfail(BAT_ERR_INVALID_ARG, "H=%lld must be > 0", H);
  if (n_seqs < 0) return gfail(BAT_ERR_INVALID_ARG, "n_seqs=%lld must be >= 0", n_seqs);
  if (n_seqs > 0 && !seq_offsets) return gfail(BAT_ERR_INVALID_ARG, "seq_offsets must be non-null");
  if (n_seqs > 0 && seq_offsets[0] < 0) return gfail(BAT_ERR_INVALID_ARG, "seq_offsets[0]=%lld is negative", seq_offsets[0]);
  for (int32_t i = 0; i < n_seqs; ++i)
    if (seq_offsets[i + 1] < seq_offsets[i])
      return gfail(BAT_ERR_INVALID_ARG, "seq_offsets not monotone at sequence %lld", i);
  const int64_t T = n_seqs ? seq_offsets[n_seqs] : 0;
  if (T > (int64_t)INT32_MAX - 256) return gfail(BAT_ERR_INVALID_ARG, "T=%lld exceeds the int32 token limit", T);
  if (num_sms <= 0) {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) == cudaSuccess && cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess &&
        n > 0)
      num_sms = n;
    else
      num_sms = 148;
    cudaGetLastError();
  }
  bat_gbla_plan* plan = new (std::nothrow) bat_gbla_plan();
  if (!plan) return gfail(BAT_ERR_OOM, "out of host memory");
  plan->n_seqs = n_seqs;
  plan->H = H;
  plan->d = d;
  plan->T = T;
  // Chunks: runs of consecutive tiles of one (sequence, head), one CTA each, one CTA per SM.
  // Their count is a whole number of waves over the SMs (about 24 tiles per chunk), dealt to the
  // pairs in proportion to their tiles (largest remainder), so every CTA gets about the same
  // number of tiles.
  std::vector<int32_t> tiles_of;
  int64_t total_tiles = 0;
  for (int32_t i = 0; i < n_seqs; ++i) {
    const int32_t tiles = (int32_t)((seq_offsets[i + 1] - seq_offsets[i] + 127) / 128);
    tiles_of.push_back(tiles);
    total_tiles += (int64_t)H * tiles;
  }
  const int64_t waves = std::max<int64_t>(1, (int64_t)std::llround((double)total_tiles / (num_sms * 24.0)));
  const int64_t target = num_sms * waves;
  std::vector<int32_t> nc_of(n_seqs, 0);
  {
    std::vector<std::pair<double, int32_t>> frac;
    int64_t given = 0;
    for (int32_t i = 0; i < n_seqs; ++i) {
      if (tiles_of[i] == 0) continue;
      const double share = total_tiles ? (double)target * tiles_of[i] / (double)total_tiles : 0.0;   // per head
      nc_of[i] = (int32_t)std::min<double>(tiles_of[i], std::max(1.0, std::floor(share)));
      given += (int64_t)H * nc_of[i];
      frac.push_back({share - std::floor(share), i});
    }
    std::sort(frac.begin(), frac.end(), [](const auto& a, const auto& b) { return a.first > b.first; });
    for (const auto& f : frac) {
      if (given + H > target) break;
      if (nc_of[f.second] < tiles_of[f.second]) {
        ++nc_of[f.second];
        given += H;
      }
    }
  }
  for (int32_t i = 0; i < n_seqs; ++i) {
    const int32_t tiles = tiles_of[i];
    if (tiles == 0) continue;
    const int32_t nc = nc_of[i];
    for (int32_t h = 0; h < H; ++h) {
      bat::GblaPair pr;
      pr.chunk0 = (int32_t)plan->chunks.size();
      pr.n_chunks = nc;
      for (int32_t k = 0; k < nc; ++k) {
        bat::GblaChunk c;
        memset(&c, 0, sizeof(c));
        c.pair = (int32_t)plan->pairs.size();
        c.head = h;
        c.seq_lo = (int32_t)seq_offsets[i];
        c.seq_hi = (int32_t)seq_offsets[i + 1];
        c.tile0 = (int32_t)((int64_t)tiles * k / nc);
        c.n_tiles = (int32_t)((int64_t)tiles * (k + 1) / nc) - c.tile0;
        plan->chunks.push_back(c);
      }
      plan->pairs.push_back(pr);
    }
  }
  const int64_t nc = (int64_t)plan->chunks.size(), np = (int64_t)plan->pairs.size();
  plan->workspace_bytes = align256(nc * kPartFloats * 4) + align256(np * 128 * 128 * 2) + align256(np * 128 * 4);
  if (!host_only && nc > 0) {
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaGetDevice(&plan->device);
    if (e == cudaSuccess) e = cudaMalloc(&plan->d_chunks, nc * sizeof(bat::GblaChunk));
    if (e == cudaSuccess) e = cudaMalloc(&plan->d_pairs, np * sizeof(bat::GblaPair));
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(plan->d_chunks, plan->chunks.data(), nc * sizeof(bat::GblaChunk), cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(plan->d_pairs, plan->pairs.data(), np * sizeof(bat::GblaPair), cudaMemcpyHostToDevice, s);
    // The host vectors live as long as the plan, so the copies may complete after this returns.
    if (e != cudaSuccess) {
      cudaFree(plan->d_chunks);
      cudaFree(plan->d_pairs);
      delete plan;
      char buf[200];
      snprintf(buf, sizeof(buf), "GBLA work list upload: %s", cudaGetErrorString(e));
      bat::set_last_error(buf);
      return e == cudaErrorMemoryAllocation ? BAT_ERR_OOM : BAT_ERR_CUDA;
    }
    plan->on_device = true;
  }
  *out = plan;
  return BAT_OK;
}

bat_status bat_gbla_plan_destroy(bat_gbla_plan* plan) {
  bat::set_last_error("");
  if (!plan) return BAT_OK;
  if (plan->on_device) {
    int cur = -1;
    cudaGetDevice(&cur);
    if (cur != plan->device) cudaSetDevice(plan->device);
    cudaFree(plan->d_chunks);
    cudaFree(plan->d_pairs);
    if (cur >= 0 && cur != plan->device) cudaSetDevice(cur);
  }
  delete plan;
  return BAT_OK;
}

size_t bat_gbla_workspace_bytes(const bat_gbla_plan* plan) { return plan ? (size_t)plan->workspace_bytes : 0; }

bat_status bat_gbla_plan_chunks(const bat_gbla_plan* plan, void* dst, size_t dst_bytes, int64_t* n_chunks) {
  bat::set_last_error("");
  if (!plan || !n_chunks) return gfail(BAT_ERR_INVALID_ARG, "plan and n_chunks must be non-null");
  *n_chunks = (int64_t)plan->chunks.size();
  const size_t need = plan->chunks.size() * sizeof(bat::GblaChunk);
  if (dst) {
    if (dst_bytes < need) return gfail(BAT_ERR_INVALID_ARG, "dst has %lld bytes, need %lld", (long long)dst_bytes, (long long)need);
    memcpy(dst, plan->chunks.data(), need);
  }
  return BAT_OK;
}

bat_status bat_gbla_forward(const bat_gbla_plan* plan, const void* q, const void* k, const void* v, const void* a,
                            const void* z, const float* conv_q, const float* conv_k, const float* conv_v,
                            const float* norm_weight, void* y, void* workspace, size_t workspace_bytes,
                            void* stream) {
  bat::set_last_error("");
  if (!plan) return gfail(BAT_ERR_INVALID_ARG, "plan must be non-null");
  if (plan->chunks.empty()) return BAT_OK;
  if (!plan->on_device) return gfail(BAT_ERR_INVALID_ARG, "the plan was built host-only and cannot run");
  if (!q || !k || !v || !a || !z || !conv_q || !conv_k || !conv_v || !norm_weight || !y)
    return gfail(BAT_ERR_INVALID_ARG, "every tensor pointer must be non-null");
  if (!al16(q) || !al16(k) || !al16(v) || !al16(z) || !al16(y) || !al16(conv_q) || !al16(conv_k) || !al16(conv_v) ||
      !al16(norm_weight) || (reinterpret_cast<uintptr_t>(a) & 1u))
    return gfail(BAT_ERR_INVALID_ARG, "q, k, v, z, y and the weights must be 16-byte aligned, a 2-byte aligned");
  if (!workspace || (int64_t)workspace_bytes < plan->workspace_bytes || !al16(workspace))
    return gfail(BAT_ERR_INVALID_ARG, "workspace needs %lld bytes (16-byte aligned), got %lld",
                 (long long)plan->workspace_bytes, (long long)workspace_bytes);
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev != plan->device)
    return gfail(BAT_ERR_INVALID_ARG, "the current device %lld is not the plan's device %lld", dev, plan->device);
  uint32_t* status = nullptr;
  cudaError_t e = bat::device_status_word(&status);
  if (e != cudaSuccess) return gfail(BAT_ERR_CUDA, "device status word lookup failed");
  const int64_t nc = (int64_t)plan->chunks.size(), np = (int64_t)plan->pairs.size();
  bat::GblaParams p;
  memset(&p, 0, sizeof(p));
  if (!encode(&p.tm_q, q, plan->T, plan->H, 136, false) || !encode(&p.tm_k, k, plan->T, plan->H, 136, false) ||
      !encode(&p.tm_v, v, plan->T, plan->H, 136, false) || !encode(&p.tm_z, z, plan->T, plan->H, 128, true) ||
      !encode(&p.tm_y, y, plan->T, plan->H, 32, true))
    return gfail(BAT_ERR_CUDA, "cuTensorMapEncodeTiled failed for a GBLA tensor");
  p.chunks = plan->d_chunks;
  p.pairs = plan->d_pairs;
  p.q = q;
  p.k = k;
  p.v = v;
  p.a = a;
  p.z = z;
  p.conv_q = conv_q;
  p.conv_k = conv_k;
  p.conv_v = conv_v;
  p.norm_w = norm_weight;
  p.y = y;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  p.part_s = reinterpret_cast<float*>(ws);
  p.state = reinterpret_cast<__nv_bfloat16*>(ws + align256(nc * kPartFloats * 4));
  p.norm_n = reinterpret_cast<float*>(ws + align256(nc * kPartFloats * 4) + align256(np * 128 * 128 * 2));
  p.H = plan->H;
  p.status = status;
  p.wait_ns = bat::wait_limit_ns();
  e = bat::launch_gbla(p, (int)nc, (int)np, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) {
    char buf[200];
    snprintf(buf, sizeof(buf), "GBLA kernel launch: %s", cudaGetErrorString(e));
    bat::set_last_error(buf);
    return BAT_ERR_CUDA;
  }
  return BAT_OK;
}

}  // extern "C"
