/*
 * bat.h - C ABI of libbat.so: bipartite prefix-shared attention on B200 (sm_100a).
 *
 * The operation (Bat: Efficient Generative Recommender Serving with Bipartite Attention,
 * lead page, sections "This paper's idea" and "Why it works"): every request holds a user
 * block and an item block of order-agnostic tokens.  One of the two blocks is the cached
 * prefix: its K/V is computed once and stored in a cache pool, and every request that
 * references it computes non-causal softmax attention for its own suffix tokens over
 *
 *     out[t, h, :] = softmax_j( scale * q[t, h, :] . [Kp ; Ks][j, h, :] ) [Vp ; Vs][j, h, :]
 *
 * where (Kp, Vp) are the rows of its cached prefix and (Ks, Vs) the rows of its own suffix.
 * There is no mask: the tokens are order-agnostic, which is why either block may serve as
 * the prefix without changing the result.
 *
 * Conventions shared by every entry point
 *   - Nothing is thrown across the ABI; each call returns a bat_status.  On failure
 *     bat_last_error() returns a message for the calling thread.
 *   - Tensors are token-major [T, H, d] with d contiguous (row stride H*d elements).
 *     They are caller-owned device memory; the library never frees them.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream).  All
 *     device work is enqueued on it; no entry point synchronises unless it says so.
 *   - bf16 tensors: d in {64, 128}; run on tcgen05 tensor cores with fp32 accumulation.
 *     fp32 tensors: d in {32, 64, 128}; run in fp32 on the CUDA cores (exact fp32 softmax).
 *   - Device pointers must be 16-byte aligned.
 */
#ifndef BAT_H_
#define BAT_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  BAT_OK = 0,
  BAT_ERR_INVALID_ARG = 1, /* a pointer, size, table or alignment was rejected */
  BAT_ERR_UNSUPPORTED = 2, /* valid arguments the library does not implement (e.g. bf16 d=32) */
  BAT_ERR_CUDA = 3,        /* a CUDA runtime or driver call failed */
  BAT_ERR_TIMEOUT = 4,     /* a kernel gave up a bounded wait and returned early */
  BAT_ERR_OOM = 5,         /* a host or device allocation of the library failed */
  BAT_ERR_DEVICE_CHECK = 6 /* debug builds only: a device-side bounds check failed */
} bat_status;

typedef enum { BAT_BF16 = 0, BAT_FP32 = 1 } bat_dtype;

/* Opaque plan: the work list of one batch, produced by the host grouping pass. */
typedef struct bat_plan bat_plan;

typedef struct {
  int32_t split_mode;        /* 0 = auto, 1 = never split, 2 = split every splittable item */
  int32_t split_chunk_tiles; /* 0 = auto; else 128-key tiles per chunk when splitting */
  int32_t num_sms;           /* 0 = the current device's SM count (148 on B200) */
  int32_t host_only;         /* 1 = build the work list on the host only (no device upload);
                                such a plan can be inspected but not run */
  int32_t reserved[4];       /* must be zero */
} bat_plan_options;

typedef struct {
  int64_t n_items;          /* work items (each: one head, up to two 128-row query tiles) */
  int64_t n_merges;         /* split query tiles whose partials are merged */
  int64_t n_slots;          /* partial slots in the workspace */
  int64_t workspace_bytes;  /* bytes bat_attention_forward needs in `workspace` */
  int64_t total_cost;       /* 128x128 score tiles over all items and heads */
  int64_t T_suf, T_cache;   /* rows the suffix tensors and the cache must have */
  int32_t R, P, H, d;
  int32_t dtype;            /* bat_dtype */
  int32_t on_device;        /* 1 when the work list was uploaded */
} bat_plan_info_t;

/*
 * bat_prefix_kv_build - pack the K/V of `num_prefixes` newly cached prefixes into the pool.
 * Section "Problem" of the lead page: the K/V of a shared prefix is computed once and
 * reused.  Prefix i's rows src[src_offsets[i] .. src_offsets[i+1]) of k_src/v_src are
 * copied to rows dst_offsets[i] .. dst_offsets[i] + len of k_cache/v_cache.
 *   k_src, v_src      device, [T_src, H, d] of dtype `dt` (read)
 *   src_offsets       HOST int64 [num_prefixes + 1], non-decreasing, src_offsets[0] >= 0
 *   dst_offsets       HOST int64 [num_prefixes], dst_offsets[i] >= 0
 *   k_cache, v_cache  device, [T_cache, H, d] of dtype `dt` (written); the caller sizes them
 * Destination ranges must not overlap each other or the sources.  Asynchronous on `stream`.
 * Errors: BAT_ERR_INVALID_ARG (null pointer, bad offsets, misalignment), BAT_ERR_CUDA.
 */
bat_status bat_prefix_kv_build(const void* k_src, const void* v_src, const int64_t* src_offsets,
                               int32_t num_prefixes, const int64_t* dst_offsets, int32_t H,
                               int32_t d, bat_dtype dt, void* k_cache, void* v_cache,
                               void* stream);

/*
 * bat_plan_create - host grouping pass over one batch of requests.
 * Lead page (Bat), section "Why it works": a hot item's cached K/V serves every user who sees
 * it and a user's cached K/V serves all of that user's requests, so the requests that read one
 * prefix are batched together and its K/V is streamed once for all of them.
 * Buckets the requests by the prefix they read, pairs their 128-row query tiles into work
 * items that stream each prefix's K/V tiles once, orders the items heaviest group first,
 * optionally splits over-long key streams (partials merged by log-sum-exp), and uploads the
 * work list to the current device on `stream` (the plan owns that device memory).
 * `dt` and `opts` go beyond the minimal interface (the pages give none): the dtype fixes
 * which kernel the plan is for, and the options expose the split policy and a host-only mode.
 *   req_prefix      HOST int32 [R]; prefix id in [0, P) or -1 for none
 *   suffix_offsets  HOST int64 [R+1]; request r owns suffix rows [so[r], so[r+1])
 *   prefix_offsets  HOST int64 [P+1]; prefix p owns cache rows [po[p], po[p+1])
 *   H, d, dt        heads, head dim and dtype the forward will run with
 *   opts            NULL for defaults
 *   out             receives the plan; release it with bat_plan_destroy
 * R = 0 and empty suffixes are valid (the forward is then a no-op for those rows).
 * The host arrays are read during the call only.
 * Errors: BAT_ERR_INVALID_ARG (non-monotone offsets, prefix id out of range, sizes beyond
 * int32 rows), BAT_ERR_UNSUPPORTED (dtype/d pair), BAT_ERR_OOM, BAT_ERR_CUDA.
 */
bat_status bat_plan_create(const int32_t* req_prefix, const int64_t* suffix_offsets,
                           const int64_t* prefix_offsets, int32_t R, int32_t P, int32_t H,
                           int32_t d, bat_dtype dt, const bat_plan_options* opts, void* stream,
                           bat_plan** out);

/*
 * bat_plan_create_prefix_side - plan for the prefix-side step: the outputs of the prefix
 * tokens themselves.  Lead page (Bat), section "Problem": the chosen prefix block's K/V is
 * computed once and cached for every request that reuses it; section "This paper's idea":
 * the tokens of a block are order-agnostic, so within its own block a token attends with no
 * mask.  Each prefix's tokens therefore attend over that prefix's tokens only: the forward
 * with no cached prefix (Lp = 0), the prefix tokens taking the place of a request's own.
 *   src_offsets  HOST int64 [num_prefixes + 1], non-decreasing: prefix i owns rows
 *                [so[i], so[i+1]) of the q/k/v tensors later passed to bat_attention_forward
 *                as q, k_suf, v_suf (k_cache = v_cache = NULL); its outputs land in the same
 *                rows of `out`.
 *   H, d, dt, opts, stream, out   as for bat_plan_create
 * Equivalent to bat_plan_create with req_prefix = -1 for every prefix and P = 0.
 * Errors: those of bat_plan_create; BAT_ERR_INVALID_ARG for num_prefixes < 0.
 */
bat_status bat_plan_create_prefix_side(const int64_t* src_offsets, int32_t num_prefixes, int32_t H,
                                       int32_t d, bat_dtype dt, const bat_plan_options* opts,
                                       void* stream, bat_plan** out);

/* Releases the plan and its device work list.  Synchronises the device first (cudaFree),
 * so work already enqueued with the plan completes.  NULL is accepted. */
bat_status bat_plan_destroy(bat_plan* plan);

/* Copies the plan's summary into *info. */
bat_status bat_plan_info(const bat_plan* plan, bat_plan_info_t* info);

/* Bytes of device workspace bat_attention_forward needs (0 when no item is split). */
size_t bat_workspace_bytes(const bat_plan* plan);

/* Copies the host copy of the work list (64-byte records, see the library's internal
 * layout) into `dst` (host) when dst_bytes >= n_items * 64.  Diagnostics and tests only. */
bat_status bat_plan_items(const bat_plan* plan, void* dst, size_t dst_bytes);
/* Same for the merge jobs (32-byte records). */
bat_status bat_plan_merges(const bat_plan* plan, void* dst, size_t dst_bytes);

/*
 * bat_attention_forward - the hot path: bipartite prefix-shared attention for every
 * suffix row of the plan's requests.  Lead page (Bat), sections "This paper's idea" and
 * "Why it works": each request's own tokens attend, with no mask, over the cached K/V of
 * its prefix block followed by its own K/V; the result equals full bidirectional attention
 * over the whole request, whichever block is the prefix.
 *   q, k_suf, v_suf   device [T_suf, H, d] of dtype dt: each request's own tokens
 *   k_cache, v_cache  device [T_cache, H, d] of dtype dt: the prefix pool (may be NULL
 *                     when T_cache = 0)
 *   scale             softmax scale; <= 0 selects 1/sqrt(d); must be finite
 *   out               device [T_suf, H, d] of dtype dt (written; rows of empty requests untouched)
 *   lse               device fp32 [H, T_suf] or NULL: natural-log log-sum-exp of the
 *                     scaled scores of each row
 *   workspace         device scratch of at least bat_workspace_bytes(plan) bytes (NULL if 0)
 * Rows outside a request's or a prefix's segment are never weighted: the kernel loads whole
 * 128-row tiles, but keys beyond a segment get weight exactly 0 and their V rows are never
 * multiplied in, so such rows may hold anything (NaN included: an unbuilt pool slot, or another
 * request's garbage) without reaching other rows' outputs.
 * One plan runs on one stream at a time: the plan holds the kernel's work-item counter, which
 * each call resets on `stream`, so two calls with the same plan whose kernels overlap (on two
 * streams) would share it and skip or repeat work.  Use one plan per concurrent stream.
 * Asynchronous on `stream`.  Device-side wait timeouts are reported by
 * bat_get_device_status.
 * Errors: BAT_ERR_INVALID_ARG (null/misaligned pointer, dtype/d differ from the plan's,
 * workspace too small, plan not on the device), BAT_ERR_CUDA.
 */
bat_status bat_attention_forward(const bat_plan* plan, const void* q, const void* k_suf,
                                 const void* v_suf, const void* k_cache, const void* v_cache,
                                 float scale, bat_dtype dt, void* out, float* lse,
                                 void* workspace, size_t workspace_bytes, void* stream);

/*
 * bat_attention_forward_noalloc - bat_attention_forward for callers that cannot allocate
 * device memory (the paper has no counterpart; this is a deployment aid).  Examples: a process
 * whose device memory is owned by another allocator that reserved the pool, or a serving loop
 * that must avoid cudaMalloc/cudaFree because they can synchronize the device.  Plans are still
 * created beforehand with bat_plan_create; this call itself allocates nothing.
 * Arguments are those of bat_attention_forward without the workspace: the split-path scratch
 * lives in a fixed 32 MiB array inside the library, held by every GPU that loads it until exit.
 *   - A plan whose bat_workspace_bytes exceeds 32 MiB is rejected: BAT_ERR_INVALID_ARG, with a
 *     message in bat_last_error() giving both sizes.
 *   - All calls on a device share that array; calls whose kernels overlap on the GPU race on
 *     it, so issue them on one stream.  It keeps the previous call's contents; nothing in it
 *     needs to start at zero.
 *   - The first call on each device resolves the array's address (with that device current);
 *     make it before any stream capture starts on that device.  The address is kept for the
 *     life of the process: after cudaDeviceReset (which unloads the library's device code) it
 *     is stale, so do not call this entry point again on a device that was reset.
 * Errors: those of bat_attention_forward, plus BAT_ERR_CUDA if the address lookup fails.
 */
bat_status bat_attention_forward_noalloc(const bat_plan* plan, const void* q, const void* k_suf,
                                         const void* v_suf, const void* k_cache, const void* v_cache,
                                         float scale, bat_dtype dt, void* out, float* lse,
                                         void* stream);

/*
 * Second workload: GBLA, gated bidirectional linear attention ("Gated Bidirectional Linear
 * Attention for Generative Retrieval", sections "Abstract" and the summary above it): linear-
 * time attention with no mask over each user history, extended by a local causal convolution
 * of q, k and v, a per-token key gate that softly forgets tokens, and a gated RMSNorm output.
 * The page gives no formulas; the library computes, per sequence and head (d = 128):
 *     x~[t] = sum_{j<4} c_x[j] * x[t-j] (zero before the sequence's first token; x = q, k, v)
 *     o[t]  = sum_s w[s] phi(q~[t]).phi(k~[s]) v~[s] / (sum_s w[s] phi(q~[t]).phi(k~[s]) + 1e-6)
 *             with phi(x) = elu(x) + 1 and the key gate w[s] = sigmoid(a[s])
 *     y[t]  = o[t] / sqrt(mean(o[t]^2) + 1e-6) * g * silu(z[t])
 * in linear time, through the sequence state S = sum_s w[s] phi(k~[s]) v~[s]^T and n.
 */
typedef struct bat_gbla_plan bat_gbla_plan;

/*
 * bat_gbla_plan_create - work list of one batch of sequences.
 *   seq_offsets  HOST int64 [n_seqs + 1], non-decreasing: sequence i owns token rows
 *                [so[i], so[i+1]) of every [T, H, ...] tensor of bat_gbla_forward
 *   H, d         heads and head width (d must be 128)
 *   num_sms      SMs to spread the chunks over (0 = the current device's count)
 *   host_only    1 = build the work list on the host only (inspectable, not runnable)
 *   out          receives the plan; release it with bat_gbla_plan_destroy
 * Errors: BAT_ERR_INVALID_ARG (bad offsets, H <= 0, T beyond int32), BAT_ERR_UNSUPPORTED
 * (d != 128), BAT_ERR_OOM, BAT_ERR_CUDA.
 */
bat_status bat_gbla_plan_create(const int64_t* seq_offsets, int32_t n_seqs, int32_t H, int32_t d,
                                int32_t num_sms, int32_t host_only, void* stream,
                                bat_gbla_plan** out);

/* Releases the plan (synchronises the device first, through cudaFree).  NULL is accepted. */
bat_status bat_gbla_plan_destroy(bat_gbla_plan* plan);

/* Device workspace bat_gbla_forward needs: the chunks' partial states and each sequence's
 * state (about 66 KB per chunk plus 33 KB per sequence and head). */
size_t bat_gbla_workspace_bytes(const bat_gbla_plan* plan);

/* Copies the work list (32-byte chunk records: pair, head, seq_lo, seq_hi, tile0, n_tiles, 2
 * pads) into dst (host) when dst is non-NULL and large enough; *n_chunks receives the count.
 * Diagnostics and tests only. */
bat_status bat_gbla_plan_chunks(const bat_gbla_plan* plan, void* dst, size_t dst_bytes,
                                int64_t* n_chunks);

/*
 * bat_gbla_forward - the GBLA layer for every token of the plan's sequences.
 *   q, k, v, z      device bf16 [T, H, 128] (z: the output gate)
 *   a               device bf16 [T, H]: key-gate logits
 *   conv_q/k/v      device fp32 [H, 4, 128]: depthwise causal convolution taps (tap j
 *                   multiplies the token j positions back)
 *   norm_weight     device fp32 [H, 128]
 *   y               device bf16 [T, H, 128] (written)
 *   workspace       device scratch of at least bat_gbla_workspace_bytes(plan) bytes
 * All device pointers 16-byte aligned (a: 2-byte).  Asynchronous on `stream`; three kernel
 * launches (state, reduce, output).  One plan and workspace run on one stream at a time.
 * Precision: the state contraction takes w*phi(k~) (scaled per chunk by a power of two so that
 * the chunk's largest gate is in (1/2, 1]) and v~ as fp16 operands, so |v~| and phi(k~) must stay
 * below 65504; the output contraction takes phi(q~) and S as bf16; accumulation is fp32.
 * Errors: BAT_ERR_INVALID_ARG (null or misaligned pointer, workspace too small, host-only
 * plan, wrong device), BAT_ERR_CUDA.
 */
bat_status bat_gbla_forward(const bat_gbla_plan* plan, const void* q, const void* k, const void* v,
                            const void* a, const void* z, const float* conv_q, const float* conv_k,
                            const float* conv_v, const float* norm_weight, void* y, void* workspace,
                            size_t workspace_bytes, void* stream);

/* Synchronises `stream`, then reports and clears the device-side status word of the
 * current device: BAT_ERR_DEVICE_CHECK if a bounds check of a debug build failed (the message
 * names the check and the offending value), BAT_ERR_TIMEOUT if a kernel abandoned a bounded
 * wait since the last call, BAT_ERR_CUDA on a CUDA error, else BAT_OK. */
bat_status bat_get_device_status(void* stream);

/* Upper bound, in nanoseconds, on every spin-wait inside the kernels (default 2e9).
 * 0 restores the default.  Diagnostics: a tiny value makes the waits run out on purpose. */
bat_status bat_set_wait_timeout_ns(uint64_t ns);

/* Message of the last failed call on this thread ("" if none). */
const char* bat_last_error(void);

/* ABI version: (major << 16) | minor. */
int32_t bat_version(void);

/* 1 in the debug build (libbat_debug.so, compiled with -DBAT_DEBUG), whose kernels check every
 * tensor-map coordinate and store index against the tensors' bounds before using it: a failed
 * check records its code and value in the device status word (reported by
 * bat_get_device_status as BAT_ERR_DEVICE_CHECK) and the access is skipped (stores) or clamped
 * into the tensor (loads).  No check traps.  0 in the normal build, which has no checks.
 * In the debug build only, the environment variable BAT_DEBUG_SHRINK_BOUNDS=n makes the checks
 * treat every tensor as n rows shorter than it is (the accesses themselves are unchanged and
 * stay inside the real tensors): a negative control showing that the checks fire. */
int32_t bat_debug_checks(void);

#ifdef __cplusplus
}
#endif
#endif /* BAT_H_ */
