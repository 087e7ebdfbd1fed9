/*
 * gqa_attn.h -- C ABI of the B200 (sm_100a) grouped-query-attention forward.
 *
 * The operation (one definition for every entry point below):
 *
 *   O = softmax( scale * Q K^T  + mask  [+ per-head sink logit] ) V
 *
 *   for batch b, query head h, query row i, with G = Hq / Hkv query heads
 *   sharing each KV head and g = floor(h / G) the KV head that h reads
 *   (contiguous grouping; AstrAI commit log, head-packing commit "pack
 *   HB = min(G, WARPS) q heads per block"):
 *     n   = kv_lens[b]  (logical length; rows n..Tkv-1 of the K/V buffers are
 *           padding and never read into the result -- nvfp4-megamoe-kernel
 *           dsv4/kernels/attention commit log, "logical vs padded N" commit)
 *     visible keys j: 0 <= j < n and, when causal, j <= n - Tq + i
 *           (causal mask aligned bottom-right against the logical length)
 *     sink[h] is one extra logit with a zero value row, in the already-scaled
 *           domain: it is never multiplied by `scale` (dsv4 attention commit
 *           log, sink commit)
 *     lse[b,h,i] = ln( sum_visible exp(s_j) + exp(sink[h]) ), natural log
 *   A row with no visible key and no sink gets O = 0 and lse = -inf.  A NaN
 *   or inf inside the first n rows of K or V makes the rows that see it NaN
 *   (IEEE arithmetic on the definition); a V value of that kind also reaches
 *   the rows of its 128-key tile that mask it by causality (their weight 0
 *   times NaN), so K/V should be finite inside the logical lengths.  The
 *   computation is tile by tile with an online-softmax (m, l, O) carry (dsv4
 *   attention commit log, multi-tile commit: running max/sum rescale, O / l
 *   once at the end); long key ranges are split over SMs and the partial
 *   (O, lse) merged by an LSE combine (AstrAI commit log, split-KV scratch
 *   validation commit; kernbench2 benches commit log, (m, l, O) merge commits).
 *
 * Layouts (all tensors contiguous, row-major, device memory unless stated):
 *   q, out   bf16  [B, Hq,  Tq,  d]
 *   k, v     bf16  [B, Hkv, Tkv, d]      Tkv = buffer capacity
 *   kv_lens  int32 [B]                   or NULL (every n = Tkv)
 *   sink     fp32  [Hq]                  or NULL (no sink)
 *   lse      fp32  [B, Hq, Tq]           or NULL (not written)
 *   o_part   fp32  [B, Hq, Tq, S, d]     (split partials, each normalised over its keys)
 *   lse_part fp32  [B, Hq, Tq, S]        (natural log; -inf for a split with no key)
 *
 * Supported: d in {64, 128, 256, 512}; Hq % Hkv == 0; 1 <= Tkv; B*Hkv*Tkv and
 * B*Hq*Tq below 2^31; every pointer 16-byte aligned.  B == 0 or Tq == 0 is a
 * valid empty call.  kv_lens values outside [0, Tkv] are clamped to that range
 * on the device and reported by gqa_get_device_error (GQA_ERR_KVLEN).
 *
 * Ownership and ordering: the caller owns every tensor.  Calls are
 * asynchronous on `stream` (a cudaStream_t; NULL = the legacy default stream)
 * and never synchronise the host.  gqa_attention_fwd keeps one scratch buffer
 * per device for its split partials (grown on the host when a larger problem
 * arrives, never freed before exit); calls on different streams of one device
 * must therefore be ordered by the caller.
 *
 * Errors: every entry point returns a gqa_status.  Argument errors are found on
 * the host before anything is launched.  Launch and attribute failures return
 * GQA_ERR_CUDA (they are never swallowed -- AstrAI commit log, dynamic shared
 * memory commit).  Waits inside the kernels are bounded: a wait that runs out
 * records GQA_ERR_TIMEOUT in a device word, the kernel returns, and
 * gqa_get_device_error reports it.
 */
#ifndef GQA_ATTN_H
#define GQA_ATTN_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st;
typedef struct CUstream_st *gqa_stream_t; /* the same handle type as cudaStream_t */

typedef enum {
    GQA_OK = 0,
    GQA_ERR_NULL = -1,        /* a required pointer is NULL */
    GQA_ERR_SHAPE = -2,       /* negative size, Hq % Hkv != 0, Tkv < 1, index overflow */
    GQA_ERR_ALIGN = -3,       /* a pointer is not 16-byte aligned */
    GQA_ERR_SPLITS = -4,      /* num_splits outside [1, GQA_MAX_SPLITS] */
    GQA_ERR_CUDA = -5,        /* a CUDA runtime/driver call failed */
    GQA_ERR_TIMEOUT = -6,     /* a bounded wait inside a kernel ran out (device-reported) */
    GQA_ERR_UNSUPPORTED = -7, /* head dim not in {64,128,256,512}, or the GPU is not sm_100 */
    GQA_ERR_KVLEN = -8,       /* a kv_lens value was outside [0, Tkv] (device-reported, clamped) */
    GQA_ERR_SCRATCH = -9,     /* the problem exceeds the scratch in place (noalloc's fixed array; graph capture) */
    GQA_ERR_PAGE = -10,       /* gqa_attention_fwd_paged: a page id outside [0, num_pages) (device-reported) */
    GQA_ERR_SMEM_ALIGN = -11  /* a kernel's dynamic shared memory was not 1024-byte aligned; it computed
                                 nothing (device-reported; an internal error, not an argument error) */
} gqa_status;

#define GQA_MAX_SPLITS 256

/*
 * The forward.  out and lse receive the attention defined above.  scale is the
 * logit multiplier (1/sqrt(d) in the usual case); causal != 0 enables the
 * bottom-right causal mask.
 *
 * CUDA graphs: once an uncaptured call of the same or larger sizes has run on
 * the device (the library's scratch is then in place), calls may be captured
 * into a graph and replayed; a captured call that would need more scratch
 * returns GQA_ERR_SCRATCH instead of allocating.  The same holds for
 * gqa_attention_fwd_paged; gqa_attention_fwd_noalloc never allocates.
 */
int gqa_attention_fwd(const void *q, const void *k, const void *v, const int32_t *kv_lens,
                      const float *sink, void *out, float *lse, int B, int Hq, int Hkv, int Tq,
                      int Tkv, int d, float scale, int causal, gqa_stream_t stream);

/*
 * The split-KV half of the forward, with the split count forced by the caller
 * (no combine, no sink).  For every query row the visible keys of its packed
 * head group are cut into num_splits contiguous ranges; split s writes the
 * attention over its range alone, normalised over that range, to
 * o_part[b,h,i,s,:] and its log-sum-exp to lse_part[b,h,i,s] (-inf, with
 * O = 0, for a range that holds no visible key).  gqa_splitkv_combine of these
 * partials (with the sink) equals gqa_attention_fwd.  Only that combination is
 * specified: where the cuts fall is an implementation choice.
 */
int gqa_attention_fwd_partial(const void *q, const void *k, const void *v, const int32_t *kv_lens,
                              int B, int Hq, int Hkv, int Tq, int Tkv, int d, float scale,
                              int causal, int num_splits, float *o_part, float *lse_part,
                              gqa_stream_t stream);

/*
 * LSE combine of S = num_splits partials per row (the merge of softmax states
 * over disjoint key sets; kernbench2 benches commit log, (m, l, O) merge and
 * its associativity):
 *   lse = ln( sum_s exp(lse_part[s]) + exp(sink[h]) ),
 *   out = sum_s exp(lse_part[s] - lse) * o_part[s]       (bf16, round to nearest)
 * sink may be NULL; lse may be NULL.  A row whose partials are all -inf and
 * that has no sink gets out = 0, lse = -inf.
 */
int gqa_splitkv_combine(const float *o_part, const float *lse_part, int num_splits,
                        const float *sink, void *out, float *lse, int B, int Hq, int Tq, int d,
                        gqa_stream_t stream);

/*
 * Sequence parallelism over a key-sharded K/V cache (kernbench2 benches commit
 * log, long-context decode commit: each device holds a slice of every
 * sequence's keys, computes the softmax state over its slice, and the states
 * are merged).  A rank that holds keys [key_offset, key_offset + shard_capacity)
 * of every sequence runs gqa_attention_fwd on its shard with the lengths below
 * (no sink, causal = 0: with one query row per head, Tq = 1, causal and
 * non-causal coincide), and gqa_combine_shards merges the ranks' results.
 */

/*
 * shard_lens[b] = clamp(kv_lens[b] - key_offset, 0, shard_capacity): how many
 * of sequence b's keys the shard holds.  kv_lens, shard_lens: int32 [B], device,
 * caller-owned.  Errors: GQA_ERR_SHAPE (negative sizes), GQA_ERR_NULL.
 */
int gqa_shard_lengths(const int32_t *kv_lens, int B, int key_offset, int shard_capacity,
                      int32_t *shard_lens, gqa_stream_t stream);

/*
 * LSE merge of per-shard results.  Shard s (0 <= s < num_shards) holds, for
 * every row (b, h, i), its output over the shard's keys, normalised over them
 * (bf16, o_shards + s * o_shard_stride elements, [B, Hq, Tq, d] contiguous) and
 * that sum's log-sum-exp (fp32, lse_shards + s * lse_shard_stride elements,
 * [B, Hq, Tq]; -inf, with output 0, where the shard holds no visible key):
 *   lse = ln( sum_s exp(lse_s) + exp(sink[h]) ),   out = sum_s exp(lse_s - lse) * O_s
 * (bf16, round to nearest).  The layout is what an all-gather of the ranks'
 * (out, lse) buffers gives.  sink may be NULL; lse may be NULL.  Requires
 * o_shards and out 16-byte aligned, o_shard_stride a multiple of 4 and, for
 * num_shards > 1, strides that keep the shards from overlapping (else
 * GQA_ERR_ALIGN / GQA_ERR_SHAPE); num_shards in [1, GQA_MAX_SPLITS].
 */
int gqa_combine_shards(const void *o_shards, long long o_shard_stride, const float *lse_shards,
                       long long lse_shard_stride, int num_shards, const float *sink, void *out,
                       float *lse, int B, int Hq, int Tq, int d, gqa_stream_t stream);

/*
 * gqa_attention_fwd over a paged K/V cache (AstrAI commit log, attention
 * commits: a KV-source policy selecting contiguous or paged K/V, page-table and
 * cache-location indices stored as int32, the paged decode address path).  The
 * pages give no cache layout; this one is the common one:
 *   k_cache, v_cache: bf16 [num_pages, Hkv, page_size, d], contiguous, caller-owned
 *                     (head-major pages: one (page, KV head) block is contiguous, so
 *                     a key tile of one head is read as whole pages);
 *   page_table:       int32 [B, max_pages] (device): logical page j of batch b is
 *                     physical page page_table[b * max_pages + j]; entries past
 *                     ceil(kv_lens[b] / page_size) are never read;
 *   kv_lens:          int32 [B] (device, required): logical lengths, each in
 *                     [0, max_pages * page_size] (else clamped, GQA_ERR_KVLEN).
 * Q, out and lse are dense as in gqa_attention_fwd; so are sink, scale, causal
 * (bottom-right against kv_lens[b]).  page_size is a power of two in [8, 1024];
 * d in {64, 128} (GQA_ERR_UNSUPPORTED otherwise).  A page id outside
 * [0, num_pages) makes the kernel read page 0 instead and report GQA_ERR_PAGE
 * through gqa_get_device_error.  Same scratch and error behaviour as
 * gqa_attention_fwd.
 */
int gqa_attention_fwd_paged(const void *q, const void *k_cache, const void *v_cache, const int32_t *page_table,
                            const int32_t *kv_lens, const float *sink, void *out, float *lse, int B, int Hq,
                            int Hkv, int Tq, int num_pages, int page_size, int max_pages, int d, float scale,
                            int causal, gqa_stream_t stream);

/*
 * gqa_attention_fwd with the K/V cache stored in FP8: OCP E4M3 bytes (sign,
 * 4-bit exponent with bias 7, 3-bit mantissa, no infinities) with one scale per
 * tensor, the storage of the AstrAI commit log's fp8 family (e4m3 quantize with
 * a per-tensor scale from the tensor's amax; the consumer multiplies back by
 * the scale).  The attention above is computed on
 *   K = value(k8) * k_scale,   V = value(v8) * v_scale.
 *   k8, v8:  uint8 [B, Hkv, Tkv, d] E4M3 bytes, contiguous, 16-byte aligned;
 *            rows past kv_lens[b] may hold anything (NaN included)
 *   k_scale, v_scale: positive finite (else GQA_ERR_SHAPE)
 * q, kv_lens, sink, out, lse, scale, causal as in gqa_attention_fwd.  Served
 * for the decode shapes of the swap-AB kernel: d = 128 with G*Tq <= 16 packed
 * query rows per KV head (GQA_ERR_UNSUPPORTED otherwise).  K/V tiles are read
 * as bytes (half the HBM traffic of bf16) and widened exactly to f16 in shared
 * memory; Q is taken to f16 (exact for |q| in [2^-14, 65504]) and P is kept in
 * f16, so the tolerance of the bf16 path against the oracle on the dequantised
 * K/V holds.  Scratch, errors and graph capture as in gqa_attention_fwd.
 */
int gqa_attention_fwd_fp8kv(const void *q, const void *k8, const void *v8, float k_scale, float v_scale,
                            const int32_t *kv_lens, const float *sink, void *out, float *lse, int B, int Hq,
                            int Hkv, int Tq, int Tkv, int d, float scale, int causal, gqa_stream_t stream);

/*
 * gqa_attention_fwd without any device allocation.  The pages have no
 * counterpart to this entry point; it exists for callers that cannot let a
 * library allocate device memory: engines that carve all of HBM into their own
 * pools at start-up, code running where an allocation (which may synchronise the
 * device) is not allowed, and hosts without a device allocator.
 *
 * Same arguments, result and validation as gqa_attention_fwd.  The split
 * partials that gqa_attention_fwd keeps in a cudaMalloc'd buffer live here in
 * one fixed array inside the library (about 21.3 MiB: 20 MiB of fp32 partial
 * rows, their lse values, 65536 merge counters and an error word), held by
 * every GPU that loads the library until the process exits.  Limits: the merge
 * counters cover at most 65536 row-blocks for head dims 64 and 128, 32768 for
 * 256 and 16384 for 512 (a row-block is 128 packed query rows of one KV head,
 * 256 when a KV head has more than 128 packed rows at head dim 64 or 128), else
 * GQA_ERR_SCRATCH; the grid uses at most as many CTAs as the array has two
 * partial slots for: 80 for head dims 256 and 512 and for head dim 128 with
 * more than 128 packed rows per KV head, one per SM otherwise.
 * The first call on a device looks up the array's device address and the SM
 * count (no allocation); make that first call outside any stream capture.
 * Every call on a device shares the array and leaves its contents behind: each
 * call clears, on its stream, the merge counters and the error word it uses,
 * and calls whose executions overlap on the GPU (on streams
 * the caller does not order) race on it.  Device-side errors (an expired bounded
 * wait, a clamped kv_lens value) are recorded in the array's error word;
 * gqa_get_device_error reads and clears it (without allocating) until the next
 * call clears it.
 */
int gqa_attention_fwd_noalloc(const void *q, const void *k, const void *v, const int32_t *kv_lens,
                              const float *sink, void *out, float *lse, int B, int Hq, int Hkv,
                              int Tq, int Tkv, int d, float scale, int causal, gqa_stream_t stream);

/*
 * Waits for `stream`, then returns (and clears) the first error a kernel of
 * this library recorded on the current device since the last call: GQA_OK,
 * GQA_ERR_TIMEOUT, GQA_ERR_KVLEN, GQA_ERR_PAGE or GQA_ERR_SMEM_ALIGN;
 * GQA_ERR_CUDA if the synchronisation itself failed.  It reads the error word
 * of the allocating entry points and that of gqa_attention_fwd_noalloc's fixed
 * array, each only if its entry points have run on the device, and allocates
 * nothing.
 */
int gqa_get_device_error(gqa_stream_t stream);

/*
 * Measurement hook (no counterpart on the pages; it only observes).  After
 * gqa_profile_begin, each gqa_attention_fwd call on the current device (up to
 * 4096 calls) records CUDA events on its own stream right before and right
 * after its kernel (one launch per call: the split-KV merge runs inside it,
 * for every head dim).
 * gqa_profile_take stops recording, waits for those events and writes, per
 * call, the kernel's duration in ms into kernel_ms[0 .. *n_calls) (kernel_ms
 * may be NULL; at most max_calls entries).
 */
int gqa_profile_begin(void);
int gqa_profile_take(float *kernel_ms, int max_calls, int *n_calls);

/* A static English description of a status code. */
const char *gqa_status_string(int status);

/* Library version, major*10000 + minor*100 + patch. */
int gqa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GQA_ATTN_H */
