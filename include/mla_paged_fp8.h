/*
 * mla_paged_fp8.h -- C ABI of the B200 (sm_100a) paged FP8-KV MLA decode library.
 *
 * The operation (one decode step of one layer):
 *   A paged KV cache holds, for every token, one MLA latent row of 576 values
 *   (512 latent + 64 rope) stored as FP8 e4m3 bytes, plus one fp32 scale per
 *   token (quantization_granularity = head_size, so one scale per token per
 *   head; Modular page "KVCacheScalesMHAOperand", description).  The cache
 *   tensors and page tables are the arguments of the Modular function
 *   "generic_get_paged_cache_with_scales" (Args):
 *     blocks  [num_blocks, kv_dim, num_layers, page_size, num_heads, head_dim]
 *     scales  [num_blocks, kv_dim, num_layers, page_size, num_heads, head_dim_granularity]
 *     cache_lengths [batch], lookup_table [batch, max_pages],
 *     max_prompt_length, max_cache_length, optional scales_lookup_table
 *     [batch, max_pages] whose ids index the scales pool when the scales are
 *     paged independently of the values.
 *   For request b, query token i < T (= max_prompt_length) and query head h:
 *     n_b   = cache_lengths[b] + T keys are stored (the step's T new tokens are
 *             already written at positions cache_lengths[b] .. n_b - 1),
 *     K[t]  = bf16_rn(f32_rn(e4m3(blocks[blk, 0, layer_idx, t % P, 0, :]) * s_t)),
 *             blk = lookup_table[b][t / P], s_t read through scales_lookup_table
 *             (or lookup_table when it is NULL) at the same slot,
 *     V[t]  = K[t][0:512],
 *     x[t]  = softmax_scale * <q[b,i,h,:], K[t]>  for t <= cache_lengths[b] + i,
 *     lse   = ln sum_t exp(x[t]),   out[b,i,h,:] = sum_t exp(x[t] - lse) V[t].
 *
 * Conventions shared by every entry point:
 *   - All tensor pointers are device pointers owned by the caller, contiguous
 *     row-major in the shapes given.  The library keeps no pointer after the
 *     call returns; the work is enqueued on `stream` and runs asynchronously,
 *     so inputs must stay alive and outputs untouched until the stream passes it.
 *   - uint32 tables are read as raw 32-bit values.
 *   - Errors are returned as mla_status_t; nothing is thrown across the ABI.
 *     mla_last_error_string() describes the last failure of the calling thread.
 *   - Device-side preconditions (page ids < pool size, cache_lengths[b] <=
 *     max_cache_length, lookup_table covering ceil(n_b / page_size) pages) are
 *     checked by the kernels: a violation skips the bad page (its rows read as
 *     stale data), sets a sticky device status word and never faults.
 *     mla_get_device_status() returns and clears that word.
 */
#ifndef MLA_PAGED_FP8_H_
#define MLA_PAGED_FP8_H_

#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MLA_OK = 0,
  MLA_ERR_INVALID_ARG = 1,   /* null pointer, bad shape, index out of range, misaligned pointer */
  MLA_ERR_UNSUPPORTED = 2,   /* valid request outside the implemented subset (see below) */
  MLA_ERR_CUDA = 3,          /* a CUDA runtime / driver call failed */
  MLA_ERR_WORKSPACE = 4,     /* workspace allocation failed */
  MLA_ERR_TIMEOUT = 5,       /* a kernel wait gave up (device status word) */
  MLA_ERR_DEVICE_BOUNDS = 6  /* a page id or length was out of range on the device (status word) */
} mla_status_t;

/* Shapes of the paged cache (the 6-D tensors of "generic_get_paged_cache_with_scales")
 * and of q.  Implemented subset: head_dim == 576, v_dim == 512, num_kv_heads == 1,
 * head_dim_granularity g in {1, 2, 3, 4, 6, 9, 12, 18, 36} (g fp32 scales per token, scale j
 * covering dims [j * 576 / g, (j + 1) * 576 / g); the KV-store step and the scale-folding decode
 * take g = 1 only), page_size a multiple of 16, kv_dim >= 1 (index 0, the latent cache, is read),
 * any num_q_heads >= 1 (processed in groups of 128). */
typedef struct {
  int32_t batch;                /* B */
  int32_t num_q_heads;          /* H */
  int32_t head_dim;             /* 576 */
  int32_t v_dim;                /* 512 */
  int32_t num_blocks;           /* leading dim of blocks */
  int32_t kv_dim;               /* second dim of blocks and scales */
  int32_t num_layers;           /* third dim of blocks and scales */
  int32_t page_size;            /* P */
  int32_t num_kv_heads;         /* num_heads of blocks / scales: 1 */
  int32_t num_scale_blocks;     /* leading dim of scales (may differ from num_blocks
                                   when scales_lookup_table != NULL) */
  int32_t head_dim_granularity; /* last dim of scales: g (1 = one scale per token) */
  int32_t max_pages;            /* second dim of lookup_table (and scales_lookup_table) */
} mla_paged_shape_t;

/*
 * mla_decode_paged_fp8 -- decode attention over the paged FP8 cache.
 *
 *   q                    bf16 [batch, max_prompt_length, num_q_heads, 576], 16-byte aligned
 *   blocks               e4m3 [num_blocks, kv_dim, num_layers, page_size, 1, 576], 16-byte aligned
 *   scales               fp32 [num_scale_blocks, kv_dim, num_layers, page_size, 1, g], 16-byte aligned;
 *                        with g > 1, dim d of a key uses its scale d / (576 / g)
 *   cache_lengths        uint32 [batch]: tokens cached before this step
 *   lookup_table         uint32 [batch, max_pages]: logical page -> block id
 *   scales_lookup_table  NULL, or uint32 [batch, max_pages]: logical page -> scale block id
 *   max_prompt_length    T >= 1, query tokens per request (uniform); host scalar
 *   max_cache_length     max_b cache_lengths[b]; host scalar, used to size the launch
 *   layer_idx            layer read from the num_layers dim, < num_layers
 *   softmax_scale        multiplies q.k before the softmax
 *   out                  bf16 [batch, max_prompt_length, num_q_heads, 512], fully overwritten
 *   lse                  fp32 [batch, max_prompt_length, num_q_heads], natural log; may be NULL
 *
 * The pages pass max_prompt_length / max_cache_length as one-element device
 * tensors; here they are host scalars so that sizing the launch needs no
 * device-to-host read.  Long requests are split across SMs and merged with an
 * LSE-weighted combine; the partial results live in a per-device workspace the
 * library allocates on the first call (and grows when a larger problem needs
 * it), so the first call on a device should not be inside stream capture.
 * Calls on different streams of one device must not overlap (they share the
 * workspace).
 */
mla_status_t mla_decode_paged_fp8(
    const void* q, const void* blocks, const float* scales,
    const uint32_t* cache_lengths, const uint32_t* lookup_table, const uint32_t* scales_lookup_table,
    uint32_t max_prompt_length, uint32_t max_cache_length, uint32_t layer_idx, float softmax_scale,
    const mla_paged_shape_t* shape, void* out, float* lse, cudaStream_t stream);

/*
 * mla_decode_paged_fp8_scale_folded -- the decode with the per-token scale folded out of the
 * keys and values (no counterpart on the reference pages; it rearranges their arithmetic).
 *
 * The key and value elements are the e4m3 values themselves, converted to bf16 exactly (every
 * e4m3 value is a bf16 value), and the scale s_t multiplies column t of the scores and column t
 * of the softmax weights:
 *     x[t] = softmax_scale * s_t * <q[b,i,h,:], e4m3(code_t)>,
 *     out[b,i,h,:] = (sum_t bf16_rn(exp(x[t] - m) * s_t) e4m3(code_t)[0:512]) / sum_t exp(x[t] - m).
 * In exact arithmetic this is attention over the unrounded products e4m3 * s_t, so it is closer to
 * that than mla_decode_paged_fp8 is; it differs from mla_decode_paged_fp8 by the fp32 and bf16
 * roundings that entry point applies to each dequantised element (well inside the decode's
 * tolerance, but not bit for bit).  The converter does no scale arithmetic, which is what makes it
 * faster.
 *
 * Arguments, ownership, workspace and errors as for mla_decode_paged_fp8, with these limits:
 * head_dim_granularity must be 1 (else MLA_ERR_UNSUPPORTED); codes 0x7F / 0xFF (e4m3 NaN) are not
 * propagated as NaN (the cache the KV-store step writes holds none).
 * The kernel uses the full 227 KB of shared memory of a CTA; mla_get_device_status reports
 * MLA_ERR_UNSUPPORTED if the runtime placed dynamic shared memory so that the kernel's layout
 * did not fit (it then writes nothing).
 */
mla_status_t mla_decode_paged_fp8_scale_folded(
    const void* q, const void* blocks, const float* scales,
    const uint32_t* cache_lengths, const uint32_t* lookup_table, const uint32_t* scales_lookup_table,
    uint32_t max_prompt_length, uint32_t max_cache_length, uint32_t layer_idx, float softmax_scale,
    const mla_paged_shape_t* shape, void* out, float* lse, cudaStream_t stream);

/*
 * mla_decode_paged_fp8_e4m3_pv -- the decode with the value product taken on the e4m3 tensor-core
 * path (kind::f8f6f4).  The pages' kernels compute the softmax-weighted sum of the value rows in
 * bf16 after dequantising them; here the value rows stay e4m3 codes and the per-token scale moves
 * into the weights, which are then represented by two e4m3 terms each.
 *
 * Scores, softmax and lse are those of mla_decode_paged_fp8 (keys dequantised to bf16 the same
 * way).  With p_t = exp(x[t] - m) and sigma = floor(log2(112 / max_t s_t)):
 *     w_t = p_t * s_t * 2^sigma,  hi_t = e4m3_rn_sat(w_t),  lo_t = e4m3_rn_sat(w_t - hi_t),
 *     out[b,i,h,:] = 2^-sigma * sum_t (hi_t + lo_t) e4m3(code_t)[0:512] / sum_t p_t.
 * hi_t + lo_t equals w_t to within 2^-8 of w_t in the normal e4m3 range (2^-10 absolute below it),
 * so out is attention over the unrounded values s_t * e4m3(code_t) up to that error per weight.
 * The kernel takes the residual in f16, lo_t = e4m3_rn_sat(f16_rn(w_t) - hi_t), which moves lo_t by
 * one step at most where the f16 rounding of w_t (2^-12 of it) crosses one of lo_t's rounding
 * boundaries; the bound above then grows by 2^-12 of w_t.
 * The largest weight lies in (56, 112], so the weights use the top of the e4m3 range.  The kernel
 * takes m and sigma per split of the keys (a running maximum of the scores that may trail the true
 * one by up to 2 in log2 units, so p_t <= 4 and w_t <= 448, and a running minimum of sigma over
 * the scales seen so far); its weights are therefore those of the formula times a factor >= 1, and
 * its result differs from a whole-row evaluation by roundings inside the same bound, not bit for
 * bit.  On the moderate-batch workload (32 requests, 1k-4k keys) it is closer to attention over the
 * unrounded values s_t * e4m3(code_t) than mla_decode_paged_fp8, whose bf16 values carry a 2^-9
 * relative rounding each.
 *
 * Arguments, ownership, workspace and errors as for mla_decode_paged_fp8_scale_folded, with the
 * same limits (head_dim_granularity 1, e4m3 NaN codes not propagated, the full 227 KB of shared
 * memory with the same MLA_ERR_UNSUPPORTED report from mla_get_device_status).
 */
mla_status_t mla_decode_paged_fp8_e4m3_pv(
    const void* q, const void* blocks, const float* scales,
    const uint32_t* cache_lengths, const uint32_t* lookup_table, const uint32_t* scales_lookup_table,
    uint32_t max_prompt_length, uint32_t max_cache_length, uint32_t layer_idx, float softmax_scale,
    const mla_paged_shape_t* shape, void* out, float* lse, cudaStream_t stream);

/* Which decode mla_decode_paged_fp8_host runs. */
enum {
  MLA_VARIANT_DECODE = 0,          /* mla_decode_paged_fp8 */
  MLA_VARIANT_SCALE_FOLDED = 1,    /* mla_decode_paged_fp8_scale_folded */
  MLA_VARIANT_E4M3_PV = 2          /* mla_decode_paged_fp8_e4m3_pv */
};

/*
 * mla_decode_paged_fp8_host -- one decode step whose per-step inputs and outputs live in host
 * memory: q, cache_lengths, lookup_table and scales_lookup_table are read from the host, out and
 * lse are written to the host; the KV cache (blocks, scales) stays in device memory.  The pages'
 * kernels take device tensors only; this entry point is the same decode with the host copies
 * folded in.
 *
 * The batch is cut into num_chunks contiguous groups of requests (0 = automatic: 4 for batch >= 64,
 * 2 for batch >= 16, else 1; at most 16).  Each group's inputs are copied to a device staging area
 * on an internal stream, decoded on `stream` (by the variant's device entry point, on the group
 * alone), and its out and lse copied back on a second internal stream, so the copies of one group
 * overlap the decode of another.  Each group is its own decode call, so the split-KV partition,
 * and with it the rounding of split rows, can differ from one call over the whole batch (within
 * the decode's tolerance; with num_chunks = 1 the results are the device entry point's bit for
 * bit).
 *
 * Arguments: as for mla_decode_paged_fp8, except that q_host [batch, max_prompt_length,
 * num_q_heads, 576] bf16, cache_lengths_host [batch], lookup_table_host and scales_lookup_table_host
 * [batch, max_pages] (the latter may be NULL) and out_host [..., 512] bf16, lse_host [batch,
 * max_prompt_length, num_q_heads] fp32 (may be NULL) are host pointers, best page-locked
 * (cudaHostAlloc / cudaHostRegister: pageable memory makes the copies synchronous), and
 * variant is one of MLA_VARIANT_*.  The caller keeps ownership of every buffer.
 *
 * Asynchronous on `stream`: when the call returns, the copies and decodes are enqueued; out_host
 * and lse_host are complete once `stream` has been synchronised (the call makes `stream` wait for
 * its last copy), and the host inputs must stay unchanged until then.  Calls must be ordered on
 * one stream per device (they share the staging area, the workspace and the internal streams).
 * The staging area grows on demand (cudaMalloc, with a device synchronisation when it is
 * replaced), so a call that grows it must not be inside stream capture.  Errors: the device entry
 * points' (checked before anything is enqueued), MLA_ERR_INVALID_ARG for a NULL host pointer, an
 * unknown variant or num_chunks outside [0, 16], MLA_ERR_WORKSPACE, MLA_ERR_CUDA.  If an error
 * occurs after copies were enqueued, the call waits for them before returning.
 */
mla_status_t mla_decode_paged_fp8_host(
    const void* q_host, const void* blocks, const float* scales,
    const uint32_t* cache_lengths_host, const uint32_t* lookup_table_host, const uint32_t* scales_lookup_table_host,
    uint32_t max_prompt_length, uint32_t max_cache_length, uint32_t layer_idx, float softmax_scale,
    const mla_paged_shape_t* shape, void* out_host, float* lse_host, int32_t variant, int32_t num_chunks,
    cudaStream_t stream);

/*
 * mla_decode_paged_fp8_noalloc -- the same decode, for callers that cannot allocate device memory
 * (for instance while a CUDA graph is being captured, under an allocator that owns the whole
 * device, or in a service that forbids allocation once it is running).  The reference pages have
 * no counterpart to this entry point.
 *
 * It takes exactly the arguments of mla_decode_paged_fp8 and produces the same results, but keeps
 * its temporary data (split plan and split-KV partial results) in one fixed device array built into
 * the library: about 42.5 MB on every GPU that loads the library, held until the process exits.
 * It never calls cudaMalloc or cudaFree.  Limits: batch * max_prompt_length *
 * ceil(num_q_heads / 128) <= 65536 (else MLA_ERR_UNSUPPORTED, with the reason in
 * mla_last_error_string), and the keys are split over at most 80 two-CTA clusters: when the
 * cluster count in force (the device's resident count, 74 on a B200, or the one set with
 * mla_set_num_clusters) is larger, the call returns MLA_ERR_UNSUPPORTED instead of changing the
 * split, so a successful call always splits the keys exactly as mla_decode_paged_fp8 does and
 * returns bit-identical results.
 * The first call on a device looks up the array's device address and sets kernel attributes; make
 * that first call before any stream capture.  All calls share the array: calls whose GPU work
 * overlaps (for example on two streams) race and corrupt each other's results, so serialise them.
 * Nothing in the array needs to start at zero: each call writes everything it later reads.
 */
mla_status_t mla_decode_paged_fp8_noalloc(
    const void* q, const void* blocks, const float* scales,
    const uint32_t* cache_lengths, const uint32_t* lookup_table, const uint32_t* scales_lookup_table,
    uint32_t max_prompt_length, uint32_t max_cache_length, uint32_t layer_idx, float softmax_scale,
    const mla_paged_shape_t* shape, void* out, float* lse, cudaStream_t stream);

/*
 * mla_gather_dequant_bf16 -- steps A and C of the decode on their own: gather every
 * stored key of every request through the page tables and dequantise it to bf16
 * with the per-token scale, K[t] = bf16_rn(f32_rn(e4m3 * s_t)).  Runs the same
 * page loader and converter code the decode kernel runs.
 *
 *   out_k  bf16 [batch, max_keys, 576]; row t of request b is written for
 *          t < cache_lengths[b] + max_prompt_length, other rows are left untouched.
 *   max_keys >= max_cache_length + max_prompt_length.
 * Other arguments as for mla_decode_paged_fp8.
 */
mla_status_t mla_gather_dequant_bf16(
    const void* blocks, const float* scales, const uint32_t* cache_lengths,
    const uint32_t* lookup_table, const uint32_t* scales_lookup_table,
    uint32_t max_prompt_length, uint32_t max_cache_length, uint32_t layer_idx,
    const mla_paged_shape_t* shape, void* out_k, uint32_t max_keys, cudaStream_t stream);

/*
 * mla_kv_store_fp8 -- the KV-store step that produces the cache the decode reads: quantise the
 * step's new tokens' latent to e4m3 with one fp32 scale per token and scatter each row into its
 * page.  The quantiser is the per-token FP8 recipe that also generates the test workloads
 * (scale amax / 448, e4m3 round to nearest with saturation); the placement is the page-table layout of
 * generic_get_paged_cache_with_scales.
 *
 * For new token i of request b, at position t = cache_lengths[b] + i (the step's tokens follow
 * the cached ones), with x its 576 bf16 values:
 *   scale = f32(max |x|) / 448 rounded to fp32 (1.0 when the row is all zero),
 *   code_d = e4m3 of f32(x_d / scale), round to nearest even, saturated to +-448,
 * written to blocks[lookup_table[b][t / P], 0, layer_idx, t % P, 0, :] and the scale to the same
 * slot of scales in block scales_lookup_table[b][t / P] when that table is given, else in the value
 * block.  Non-finite inputs are not supported.
 *
 *   latent          bf16 [batch, num_new_tokens, 576], contiguous, 16-byte aligned, device memory.
 *   cache_lengths   uint32 [batch] device; positions must satisfy t / P < max_pages.
 *   lookup_table, scales_lookup_table   as for mla_decode_paged_fp8; the pages must already be
 *                   assigned (this call writes into them, it does not allocate pages).
 *   blocks, scales  the cache, written in place (only the rows of the new tokens, kv_dim 0).
 *   shape           as for mla_decode_paged_fp8 (head_dim 576, num_kv_heads 1,
 *                   head_dim_granularity 1; num_q_heads, v_dim and max_prompt_length are not used).
 * Asynchronous on `stream`.  A page id past the pool or a position past max_pages is skipped on
 * the device and reported by mla_get_device_status as MLA_ERR_DEVICE_BOUNDS.  Two new tokens that
 * map to the same slot race (the caller's tables must not do that).  batch = 0 or
 * num_new_tokens = 0 is a no-op.
 */
mla_status_t mla_kv_store_fp8(
    const void* latent, const uint32_t* cache_lengths, const uint32_t* lookup_table,
    const uint32_t* scales_lookup_table, uint32_t num_new_tokens, uint32_t layer_idx,
    const mla_paged_shape_t* shape, void* blocks, float* scales, cudaStream_t stream);

/*
 * mla_merge_lse_parts_bf16 -- the merge step of context parallelism (no counterpart on the
 * reference pages): when every rank decodes a contiguous, page-aligned range of each request's
 * keys (mla_decode_paged_fp8 on a page table that lists only those pages), the ranks' results are
 * exchanged and merged here.  For each of `rows` rows (request, query token, head) and parts
 * r = 0 .. num_parts - 1:
 *     lse[row] = ln sum_r e^{lses[r][row]},   out[row] = sum_r e^{lses[r][row] - lse[row]} outs[r][row]
 * which is the softmax attention over the union of the parts' keys.  A part with lse = -inf (no keys)
 * is skipped; a row with no non-empty part gets out = 0 and lse = -inf.
 *
 *   outs   bf16 [num_parts, rows, 512], device, 16-byte aligned (each part's decode `out`)
 *   lses   fp32 [num_parts, rows], device (each part's decode `lse`, natural log)
 *   out    bf16 [rows, 512], device, 16-byte aligned, fully overwritten; may not alias outs
 *   lse    fp32 [rows] or NULL
 * Asynchronous on `stream`; rows = 0 is a no-op.  Errors: MLA_ERR_INVALID_ARG (NULL or misaligned
 * pointers, num_parts < 1), MLA_ERR_CUDA.
 */
mla_status_t mla_merge_lse_parts_bf16(const void* outs, const float* lses, int32_t num_parts, int64_t rows,
                                      void* out, float* lse, cudaStream_t stream);

/*
 * mla_set_num_clusters -- test and tuning hook: fix the number of 2-CTA clusters
 * the decode splits the keys over (0 restores the default, one per resident
 * cluster slot of the device).  Process-wide.  Smaller values make fewer, longer
 * pieces; values above the resident count run in several waves.
 */
mla_status_t mla_set_num_clusters(int32_t num_clusters);

/*
 * mla_set_timing_events -- measurement hook: when both events are non-NULL, every later
 * mla_decode_paged_fp8 call on this thread records `before` on its stream right before
 * launching the decode kernel and `after` right after it, so that the caller can time that
 * kernel alone (cudaEventElapsedTime).  Pass NULL, NULL to stop.  The events stay owned by
 * the caller.
 */
mla_status_t mla_set_timing_events(cudaEvent_t before, cudaEvent_t after);

/*
 * mla_set_wait_limit_ns -- bound of every wait inside the decode kernel (the roles of a CTA pair
 * hand tiles to each other through mbarriers).  A wait that runs out makes every role of the pair
 * stop, drain its own copies and MMAs and return; the call's results are then undefined and the
 * next mla_get_device_status returns MLA_ERR_TIMEOUT.  Default 2 s; accepted range [1 ms, 60 s]
 * (else MLA_ERR_INVALID_ARG).  Process-wide; applies to calls made after it.
 */
mla_status_t mla_set_wait_limit_ns(uint64_t ns);

/*
 * mla_debug_withhold_arrival_once -- test hook for the timeout path: in the next decode call (of
 * any entry point) the Q loader of CTA 1 of the first cluster withholds its arrival on the first
 * unit's Q-ready barrier, so the Q.K^T issuer's wait runs out after the wait limit.  The call
 * returns normally, its results are undefined, and mla_get_device_status then reports
 * MLA_ERR_TIMEOUT; the device stays usable.  No reference page has a counterpart.
 */
mla_status_t mla_debug_withhold_arrival_once(void);

/* Number of clusters the next decode on the current device will use. */
int32_t mla_get_num_clusters(void);

/* Text of the last error on the calling thread ("" if none). */
const char* mla_last_error_string(void);

/*
 * mla_get_device_status -- synchronises `stream`, then returns and clears the
 * sticky device status word of the current device: MLA_OK, MLA_ERR_DEVICE_BOUNDS
 * or MLA_ERR_TIMEOUT.
 */
mla_status_t mla_get_device_status(cudaStream_t stream);

/* Frees the workspace of every device this thread's process used (synchronises them). */
mla_status_t mla_release_workspace(void);

/* Library version, e.g. "0.1.0". */
const char* mla_version(void);

#ifdef __cplusplus
}
#endif
#endif /* MLA_PAGED_FP8_H_ */
