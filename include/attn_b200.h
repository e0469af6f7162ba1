/*
 * attn_b200.h -- C ABI of libattn_b200.so: fused grouped-query attention
 * forward for NVIDIA B200 (sm_100a).
 *
 * Operation ("带你了解Attention,从MHA到DeepSeek" section 1.2; "GQA和MLA详解"
 * sections 1-3; "Full 路线：保留 softmax，压缩 K/V 表示" sections 三 and 4.3):
 *
 *   out[b,h,i,:] = sum_j softmax_j( scale * q[b,h,i,:] . k[b,h/G,j,:] ) v[b,h/G,j,:]
 *   lse[b,h,i]   = ln sum_j exp( scale * q[b,h,i,:] . k[b,h/G,j,:] )
 *
 * with G = Hq / Hkv query heads per K/V head (G = Hq is MQA, G = 1 is MHA;
 * query head h reads kv head h / G, as repeat_interleave does), j running
 * over the visible keys of sequence b: j < skv[b], and with `causal` set,
 * j <= i + skv[b] - Sq (bottom-right alignment: a single decode query sees
 * every key).  A row with no visible key yields out = 0 and lse = -inf.
 *
 * Absorbed MLA decode ("Full 路线" section 4.3: W_UK folded into the query,
 * the cache holds rows [c_kv (512) | k_pe (64)]) is the same call with
 * d_k = 576, d_v = 512, Hkv = 1 and v pointing at the same rows as k (the
 * first 512 columns): each cached row then comes from DRAM about once (its
 * first 512 columns are read again as V from L2), and all query heads of a
 * sequence share it (pairs of SMs, 128 heads per pair).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Tensors are row-major [B, H, S, d] addressed with element strides
 *   (attn_strides_t: b, h, s); the innermost (d) stride is 1.  All device
 *   pointers must be 16-byte aligned and every stride a multiple of 8
 *   elements (16 bytes), which tensor-memory-access (TMA) copies require.
 * - q: [B, Hq, Sq, d_k]; k: [B, Hkv, >= max_skv, d_k]; v: [B, Hkv,
 *   >= max_skv, d_v]; out: [B, Hq, Sq, d_v] (same element type as q);
 *   lse: [B, Hq, Sq] fp32, contiguous, may be NULL.
 * - Key rows at or past skv[b] (up to max_skv) are never read: they may
 *   hold anything, e.g. memory not yet written by a growing cache (a
 *   sequence's partial last tile is fetched as the tile-sized window that
 *   ends at its last key).
 * - Ownership: the caller owns every buffer (q, k, v, out, lse, skv,
 *   workspace).  The library allocates no device memory and never
 *   synchronises the stream inside attn_fwd; all work is enqueued on
 *   `cuda_stream` (a cudaStream_t; NULL = the legacy default stream).
 * - Errors: argument problems are reported before anything is launched;
 *   device-side waits that exceed their time limit set a device error word
 *   read by attn_last_device_error().
 *
 * Supported shapes: (d_k, d_v) in {(128,128), (512,512)} for any Sq;
 * (576, 512) -- absorbed MLA over [c_kv | k_pe] rows -- for decode (Sq == 1);
 * (192, 128) -- MLA prefill in its expanded (MHA) form -- for Sq > 1.
 * Sq == 1, and Sq in {2, 4, 8, 16} at d_k in {128, 512} (extend / speculative
 * decoding against a cache), take the split-KV decode path; other Sq > 1 the
 * prefill kernel.  Element type bf16 or fp16.  Anything else returns
 * ATTN_EUNSUPPORTED; there is no fallback.
 */
#ifndef ATTN_B200_H
#define ATTN_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  ATTN_OK = 0,
  ATTN_EINVAL = 1,        /* bad pointer, size, stride or alignment            */
  ATTN_EUNSUPPORTED = 2,  /* valid request outside the supported shapes        */
  ATTN_EWORKSPACE = 3,    /* workspace missing or smaller than required        */
  ATTN_ECUDA = 4,         /* a CUDA runtime/driver call or launch failed       */
  ATTN_ETIMEOUT = 5,      /* a device-side wait gave up (see attn_last_device_error) */
  ATTN_EOVERFLOW = 6,     /* attn_cache_append found a full sequence (see attn_last_device_error) */
  ATTN_EINDEX = 7         /* attn_gather_rows met a position outside its sequence (ditto) */
} attn_status_t;

typedef enum { ATTN_BF16 = 0, ATTN_FP16 = 1 } attn_dtype_t;

/* Element strides of a [B, H, S, d] tensor; the d stride is always 1. */
typedef struct {
  int64_t b, h, s;
} attn_strides_t;

/* What attn_fwd will launch for a problem (host-side plan, no GPU needed). */
typedef struct {
  int path;            /* 0 = prefill kernel, 1 = split-KV decode + combine      */
  int heads_per_cta;   /* decode: (query head x query) columns packed into one
                          CTA's MMA N (MLA: heads per pair of CTAs)              */
  int head_blocks;     /* decode: CTAs per key range along the group's G * Sq
                          columns                                                */
  int kv_ranges;       /* decode: equal ranges the concatenated key tiles of all
                          (sequence, kv head) pairs are cut into, one persistent
                          CTA per range and head block                           */
  int64_t partials;    /* decode: partial-result slots (kv_ranges + B * Hkv)    */
  int dv_parts;        /* prefill: CTAs sharing one q tile, each owning d_v/dv_parts columns */
  int64_t grid_ctas;   /* CTAs of the main kernel (persistent: at most one wave) */
  size_t workspace_bytes;
} attn_plan_t;

/*
 * Plan a call.  `num_sms` <= 0 means "ask the current device" (148 if no
 * device is visible).  Pure host computation; returns ATTN_EINVAL /
 * ATTN_EUNSUPPORTED under the same rules as attn_fwd.
 * Source: "GQA和MLA详解" section 1 (prefill is the quadratic T x T phase,
 * decode reads the whole cache once per step and is bandwidth-bound).
 */
attn_status_t attn_plan(int B, int Hq, int Hkv, int Sq, int max_skv, int d_k, int d_v,
                        attn_dtype_t dtype, int num_sms, attn_plan_t* plan);

/*
 * Workspace bytes attn_fwd needs for this problem on the current device
 * (0 for prefill).  Decode stores partial outputs (fp32 [partials, G * Sq,
 * d_v]) and partial LSEs (fp32 [partials, G * Sq]) there, one slot per piece of a
 * (sequence, kv head) pair that falls in one key range.  Returns 0 for
 * arguments attn_plan rejects.
 */
size_t attn_workspace_bytes(int B, int Hq, int Hkv, int Sq, int max_skv, int d_k, int d_v);

/*
 * The forward pass (definition at the top of this file).
 *   skv_per_seq: device pointer, int32 [B], 0 <= skv[b] <= max_skv (not
 *                checked on the device).
 *   max_skv:     host value, the row extent of k and v (>= 1).
 *   scale:       > 0, multiplies q.k before the softmax (1/sqrt(d_k) for plain
 *                attention; 1/sqrt(192) for DeepSeek-V3 MLA, whose score
 *                scale follows the un-absorbed head width).
 *   causal:      0 or 1 (bottom-right alignment, see above).
 *   workspace:   device buffer of at least attn_workspace_bytes(...) bytes,
 *                16-byte aligned (may be NULL when that is 0).  Concurrent
 *                calls must not share a workspace.
 * Returns ATTN_OK once the kernels are enqueued.
 */
attn_status_t attn_fwd(const void* q, const void* k, const void* v, void* out, float* lse,
                       int B, int Hq, int Hkv, int Sq,
                       const int32_t* skv_per_seq, int max_skv,
                       int d_k, int d_v, float scale, int causal, attn_dtype_t dtype,
                       attn_strides_t sq, attn_strides_t sk, attn_strides_t sv, attn_strides_t so,
                       void* workspace, size_t workspace_bytes, void* cuda_stream);

/*
 * The two steps attn_fwd enqueues for a decode-path problem (plan path 1), callable
 * separately with attn_fwd's arguments (for timing each kernel, or for
 * overlapping the merge with other work):
 *   attn_decode_partial  -- one persistent CTA per key range and head block
 *                           attends over each piece of a (sequence, kv head)
 *                           pair in its range and writes a normalised partial
 *                           output and its LSE into the workspace;
 *   attn_decode_combine  -- merges the pieces of each (b, h, query) in range order:
 *                           L = ln sum_s exp(lse_s), out = sum_s exp(lse_s - L) o_s
 *                           ("GQA和MLA详解" section 4: a fixed reduction order keeps
 *                           the result bitwise reproducible).
 * Same validation and errors as attn_fwd; ATTN_EINVAL for prefill-path problems.  The
 * combine step reads what the partial step wrote into the same workspace.
 */
attn_status_t attn_decode_partial(const void* q, const void* k, const void* v, void* out,
                                  float* lse, int B, int Hq, int Hkv, int Sq,
                                  const int32_t* skv_per_seq, int max_skv, int d_k, int d_v,
                                  float scale, int causal, attn_dtype_t dtype, attn_strides_t sq,
                                  attn_strides_t sk, attn_strides_t sv, attn_strides_t so,
                                  void* workspace, size_t workspace_bytes, void* cuda_stream);
attn_status_t attn_decode_combine(const void* q, const void* k, const void* v, void* out,
                                  float* lse, int B, int Hq, int Hkv, int Sq,
                                  const int32_t* skv_per_seq, int max_skv, int d_k, int d_v,
                                  float scale, int causal, attn_dtype_t dtype, attn_strides_t sq,
                                  attn_strides_t sk, attn_strides_t sv, attn_strides_t so,
                                  void* workspace, size_t workspace_bytes, void* cuda_stream);

/*
 * attn_fwd without a workspace argument, for callers that cannot allocate
 * device memory (the pages have no counterpart: this is a library concern).
 * Examples: a plugin run by a host framework that owns all device memory
 * and gives plugins no allocator, or a latency-critical loop in which
 * cudaMalloc's implicit device-wide synchronisation is not acceptable.
 *
 * Scratch comes from a buffer of ATTN_NOALLOC_SCRATCH_BYTES compiled into
 * the library (held on every GPU that loads the library until the process
 * exits); the call itself allocates nothing.  Problems whose scratch
 * (attn_workspace_bytes) exceeds that size return ATTN_EWORKSPACE before
 * anything is enqueued.  The device that holds the tensors and owns
 * `cuda_stream` must be the calling thread's current device: the buffer
 * and the launch plan are taken from the current device.  The first call
 * on each device looks up the buffer's device address (cudaGetSymbolAddress,
 * that device current), and so does the first call after the device's
 * context has been replaced (cudaDeviceReset); make that first call before
 * any stream capture.  All calls share the buffer: calls that overlap on
 * the GPU (concurrent streams or host threads) race, so serialise them.
 * Otherwise the same arguments, semantics and errors as attn_fwd.
 */
#define ATTN_NOALLOC_SCRATCH_BYTES (32u << 20)
attn_status_t attn_fwd_noalloc(const void* q, const void* k, const void* v, void* out,
                               float* lse, int B, int Hq, int Hkv, int Sq,
                               const int32_t* skv_per_seq, int max_skv, int d_k, int d_v,
                               float scale, int causal, attn_dtype_t dtype, attn_strides_t sq,
                               attn_strides_t sk, attn_strides_t sv, attn_strides_t so,
                               void* cuda_stream);

/*
 * Synchronises `cuda_stream`, then reads and clears the current device's
 * error word.  ATTN_OK if no kernel of this library reported a problem
 * since the last call, ATTN_ETIMEOUT if a device-side wait gave up (the
 * outputs of that launch are undefined), ATTN_EOVERFLOW if attn_cache_append
 * met a full sequence, ATTN_EINDEX if attn_gather_rows met a position outside
 * its sequence, ATTN_ECUDA if the stream itself reports an error.
 */
attn_status_t attn_last_device_error(void* cuda_stream);

/*
 * Append the new token's cached row(s) before a decode step ("Full 路线"
 * section 三: past_key_value.update, then attention over the whole cache;
 * sections 4.2-4.3: in MLA the cached row is [c_kv | k_pe]).  For every
 * sequence b whose length skv[b] < max_skv, and every kv head h, copies
 * k_new[b, h, :] (d_k elements) to k_cache[b, h, skv[b], :] and
 * v_new[b, h, :] (d_v elements) to v_cache[b, h, skv[b], :], then sets
 * skv[b] += 1 -- all on `cuda_stream`, so an attn_fwd enqueued after it on
 * the same stream attends over the new key as well.
 * - k_cache/v_cache: [B, Hkv, max_skv, d] with element strides sk / sv
 *   (innermost contiguous); k_new/v_new: [B, Hkv, 1, d] with strides skn /
 *   svn (the s stride is ignored).  skv_per_seq: device int32 [B], updated.
 * - MLA latent cache: pass v_cache == k_cache (or NULL); only the K row (the
 *   whole [c_kv | k_pe] row, d_k = 576) is written and v_new is ignored.
 * - A sequence already holding max_skv keys is left unchanged and bit 1 of
 *   the device error word is set: attn_last_device_error then returns
 *   ATTN_EOVERFLOW.
 * - Errors before launch: ATTN_EINVAL (null or misaligned pointers, strides
 *   or d not multiples of 8 elements, bad dtype); ATTN_ECUDA on a launch error.
 * The pages have no counterpart beyond the cache update they call.
 */
attn_status_t attn_cache_append(void* k_cache, void* v_cache, const void* k_new, const void* v_new,
                                int32_t* skv_per_seq, int B, int Hkv, int max_skv, int d_k,
                                int d_v, attn_dtype_t dtype, attn_strides_t sk, attn_strides_t sv,
                                attn_strides_t skn, attn_strides_t svn, void* cuda_stream);

/*
 * Top-k sparse decode in the DSA style ("带你了解Attention,从MHA到DeepSeek"
 * section 5.1: an indexer -- not part of this library -- selects the top-k
 * cached entries for each new token; attention then runs over those only):
 * copies, for every sequence b and head h < H, the rows at the selected
 * positions idx[b * idx_stride + t], t < n_sel[b] (at most topk), of
 * src [B, H, >= skv[b], d] into dst [B, H, >= topk, d] in selection order,
 * and writes dst_len[b] = n_sel[b].  An attn_fwd on (q, dst, dst_len) on the
 * same stream is then attention over the selected keys (for MLA pass dst as
 * both k and v with d = 576).  A position outside [0, skv[b]) yields a zero
 * row and sets bit 2 of the device error word (ATTN_EINDEX from
 * attn_last_device_error).
 * - idx, n_sel, skv_per_seq, dst_len: device int32; src/dst: element
 *   strides s_src / s_dst (innermost contiguous), 16-byte aligned, d a
 *   multiple of 8.  Errors before launch: ATTN_EINVAL; ATTN_EUNSUPPORTED for
 *   B or H above 65535; ATTN_ECUDA on a launch error.
 */
attn_status_t attn_gather_rows(const void* src, void* dst, const int32_t* idx,
                               const int32_t* n_sel, const int32_t* skv_per_seq, int32_t* dst_len,
                               int B, int H, int topk, int d, attn_dtype_t dtype,
                               attn_strides_t s_src, attn_strides_t s_dst, int64_t idx_stride,
                               void* cuda_stream);

/*
 * Top-k sparse absorbed-MLA decode in one pass (the same passage: attention
 * over the cached entries an indexer selected): out[b, h] = attention of
 * q[b, h] over the rows at positions idx[b * idx_stride + t], t < n_sel[b],
 * of the latent cache [B, 1, >= skv[b], 576] (k = whole rows, v = their first
 * 512 columns), equal to attn_gather_rows followed by attn_fwd, but the rows
 * are copied straight from the cache into the decode kernel's shared memory,
 * so each selected byte crosses HBM once.
 * - q [B, Hq, 1, 576], out [B, Hq, 1, 512], lse [B, Hq, 1] or NULL; element
 *   strides sq / sc (cache) / so, innermost contiguous, 16-byte aligned.
 * - idx, n_sel, skv_per_seq: device int32; 0 <= n_sel[b] <= topk (not
 *   checked on the device); idx_stride >= topk.  A position outside
 *   [0, skv_per_seq[b]) reads as a zero row and sets bit 2 of the device
 *   error word (ATTN_EINDEX from attn_last_device_error).
 * - max_skv: row extent of the cache; workspace: attn_workspace_bytes(B, Hq,
 *   1, 1, topk, 576, 512) bytes, 16-byte aligned, owned by the caller.
 * - Errors before launch: ATTN_EINVAL, ATTN_EUNSUPPORTED (d_k != 576 or
 *   d_v != 512, or what attn_plan refuses), ATTN_EWORKSPACE, ATTN_ECUDA.
 */
attn_status_t attn_topk_fwd(const void* q, const void* cache, void* out, float* lse, int B, int Hq,
                            const int32_t* idx, int64_t idx_stride, const int32_t* n_sel,
                            const int32_t* skv_per_seq, int topk, int max_skv, int d_k, int d_v,
                            float scale, attn_dtype_t dtype, attn_strides_t sq, attn_strides_t sc,
                            attn_strides_t so, void* workspace, size_t workspace_bytes,
                            void* cuda_stream);

/* Bound on every device-side wait of launches made after this call, in
 * nanoseconds of %globaltimer (process-wide; 0 restores the default of 2 s).
 * Returns the previous bound.  A diagnostic: a bound far below a kernel's
 * normal waiting times makes its waits give up, so the error path (abort,
 * drain, ATTN_ETIMEOUT from attn_last_device_error) can be exercised without
 * any fault.  The pages have no counterpart.  Not synchronised with launches
 * running on other host threads. */
uint64_t attn_set_wait_timeout_ns(uint64_t ns);

/* Static, human-readable name of a status code. */
const char* attn_status_str(attn_status_t status);

/* Library version, e.g. "0.1.0". */
const char* attn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* ATTN_B200_H */
