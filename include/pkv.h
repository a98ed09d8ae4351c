/*
 * pkv.h -- libpkv, the C ABI of one in-flight-batched decode step over a
 * paged KV cache on a B200 GPU (sm_100a).
 *
 * The step, for every request b of a batch of requests of different lengths
 * ("Scaling TensorRT-LLM: Kernel Fusion and Inflight Batching in
 * Production", section "Static vs. Dynamic vs. Inflight"):
 *   1. rotary embedding of the new token's q (all query heads) and k at
 *      position L_b = seq_lens[b] (same page, section "What Gets Fused",
 *      RoPE bullet);
 *   2. append of the rotated k and the raw v into slot L_b % P of physical
 *      page block_tables[b][L_b / P] (same page, section "The Paged
 *      KV-Cache"; "TensorRT-LLM Guide: High-Throughput GPU Inference
 *      Engine", section "2. Paged KV Cache & Memory Virtualization");
 *   3. grouped-query attention of the single new query over all n_b = L_b + 1
 *      tokens of the request, each KV element read once for the G = Hq/Hkv
 *      query heads that share it ("TensorRT-LLM Guide", section "3. Custom
 *      Fused Attention Kernels: FMHA and XQA"), softmax kept on chip (first
 *      page, section "What Gets Fused", Attention bullet).
 * Optional E4M3 KV cache with one fp32 scale per (page, kv head)
 * ("TensorRT-LLM Guide", section "4. Native FP8 Quantization on NVIDIA
 * Hopper & Blackwell").
 *
 * Definitions used (the pages name the operations but give no formula):
 *   RoPE: rotate-half pairs (i, i + d/2), theta_i = rope_base^(-2i/d),
 *         x_i' = x_i cos(p theta_i) - x_{i+d/2} sin(p theta_i),
 *         x_{i+d/2}' = x_{i+d/2} cos(p theta_i) + x_i sin(p theta_i);
 *   attention: o_h = softmax(q_h K^T / sqrt(d)) V over the request's tokens
 *         in logical order, K/V of kv head h / G (contiguous groups);
 *   fp8 store: code = E4M3_RNE_satfinite(fl32(x / scale[page][kvh]));
 *   fp8 load: value = code * scale[page][kvh].
 *
 * Layouts (all row-major, all caller-owned device memory):
 *   q, out          [batch][Hq][d]        bf16
 *   k_new, v_new    [batch][Hkv][d]       bf16
 *   k_pool, v_pool  [num_pages][Hkv][P][d] bf16, or uint8 E4M3 codes
 *   k_scale,v_scale [num_pages][Hkv]      fp32 (fp8 pools only; else NULL)
 *   block_tables    [batch][bt_stride]    int32 physical page ids
 *   seq_lens        [batch]               int32, L_b = tokens cached BEFORE
 *                                         the step; the step attends L_b + 1
 * Every pointer must be 16-byte aligned.
 *
 * Ownership and ordering: the library never allocates, frees or keeps caller
 * tensors.  A context owns its workspace (split partials, the split geometry
 * passed from the attention kernel to its combine, a device error word), allocated in pkv_create and
 * freed in pkv_destroy; use one context from one stream at a time.  Calls are
 * asynchronous and stream-ordered: they validate on the host, enqueue, and
 * return.  pkv_rope_append writes q (in place) and exactly batch * Hkv slots
 * of each pool; pkv_decode_attn writes only out.  The caller allocates the
 * page the new token lands in before the step; block-table entries past
 * ceil(n_b / P) are never read.
 *
 * Beyond the step (each declared below with its own contract):
 *   pkv_decode_step                                  both parts of the step in
 *       one call, the attention overlapping the end of the append;
 *   pkv_rope_append_tokens / pkv_decode_attn_tokens  several new tokens per
 *       request, the same count for all (speculative verification);
 *   pkv_rope_append_varlen / pkv_decode_attn_varlen  a count per request,
 *       packed (chunked prefill mixed with decode);
 *   pkv_qkv_rope_append, pkv_qkv_pack_weight         the QKV projection of
 *       the new tokens on the tensor cores fused with RoPE and the append;
 *   pkv_table_sync                                   the device side of the
 *       host page allocator of pkv_pages.h;
 *   pkv_decode_attn_noalloc                          the attention without a
 *       context (no allocation);
 *   pkv_set_workers, pkv_set_tail_chunks, pkv_set_qkv_split, pkv_set_prefill_rows,
 *   pkv_qkv_launch_shape, pkv_workspace_bytes        tuning and inspection.
 *
 * Errors: host-side checks return PKV_ERR_INVALID_ARG / PKV_ERR_UNSUPPORTED
 * and launch nothing.  A failed launch returns PKV_ERR_CUDA.  Range errors
 * found on the device (a page id outside [0, num_pages), or L_b + 1 larger
 * than bt_stride * P) skip the affected request or tile and set a sticky
 * device error word, which pkv_check_device_error reads; no call traps.
 * C++ exceptions never cross this ABI.
 */
#ifndef PKV_H
#define PKV_H

#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct pkv_ctx pkv_ctx;

typedef enum {
    PKV_OK = 0,
    PKV_ERR_INVALID_ARG = 1,    /* NULL / misaligned pointer, bad size, bad config */
    PKV_ERR_UNSUPPORTED = 2,    /* valid but not built: head_dim, page size, group size */
    PKV_ERR_CUDA = 3,           /* a CUDA runtime call or launch failed */
    PKV_ERR_OOM = 4,            /* workspace allocation failed */
    PKV_ERR_DEVICE_BOUNDS = 5,  /* device saw a page id or length out of range */
    PKV_ERR_DEVICE_TIMEOUT = 6  /* a bounded wait inside a kernel gave up */
} pkv_status;

typedef enum { PKV_KV_BF16 = 0, PKV_KV_FP8_E4M3 = 1 } pkv_kv_dtype;

/* Shapes fixed at create time, like an engine built for one model and
 * limits ("TensorRT-LLM", section "What the build step is for"). */
typedef struct {
    int num_q_heads;          /* Hq; a multiple of num_kv_heads */
    int num_kv_heads;         /* Hkv; G = Hq / Hkv must be 1..8 */
    int head_dim;             /* d: 64 or 128 */
    int page_size;            /* P: 16, 32 or 64 tokens */
    pkv_kv_dtype kv_dtype;    /* pool element type */
    double rope_base;         /* > 1, e.g. 10000 or 500000 */
    int max_batch;            /* largest batch a call may pass (<= 8192) */
    int max_blocks_per_seq;   /* largest bt_stride a call may pass */
    int num_pages;            /* physical pages in each pool */
} pkv_config;

/* Validates cfg, binds the context to the current CUDA device and allocates
 * its workspace.  *out is set only on PKV_OK.  Validation happens before any
 * CUDA call, so a bad cfg is reported without touching the device. */
pkv_status pkv_create(const pkv_config* cfg, pkv_ctx** out);

/* Step part 1 (RoPE + append).  Rotates q in place and k_new at position
 * L_b, stores rotated k and raw v into slot L_b % P of page
 * block_tables[b * bt_stride + L_b / P].  bf16 pools: k is rounded to bf16
 * (nearest even) from the exact rotation, v copied bit for bit.  fp8 pools:
 * the E4M3 store above with k_scale / v_scale of that page and kv head.
 * batch == 0 is a no-op. */
pkv_status pkv_rope_append(pkv_ctx* ctx, void* q, const void* k_new, const void* v_new,
                           void* k_pool, void* v_pool,
                           const float* k_scale, const float* v_scale,
                           const int32_t* block_tables, int bt_stride,
                           const int32_t* seq_lens, int batch, cudaStream_t stream);

/* Step part 2 (decode attention).  q holds the rotated queries written by
 * pkv_rope_append; seq_lens is the same L_b, and n_b = L_b + 1 tokens are
 * attended (the new one included).  out[b][h][:] = bf16(o_h).  Work is split
 * over all SMs by token ranges (optionally with a dynamic tail, see
 * pkv_set_tail_chunks); partial results of a (request, kv head) cut between
 * ranges or chunks are merged by log-sum-exp in a second, small kernel
 * enqueued right after on the same stream.  That kernel also resets the
 * context's chunk counter; if this call returns PKV_ERR_CUDA the context
 * should be destroyed, not reused.
 * batch == 0 is a no-op. */
pkv_status pkv_decode_attn(pkv_ctx* ctx, const void* q, const void* k_pool, const void* v_pool,
                           const float* k_scale, const float* v_scale,
                           const int32_t* block_tables, int bt_stride,
                           const int32_t* seq_lens, int batch, void* out,
                           cudaStream_t stream);

/* Several new tokens per request: the verification pass of speculative
 * decoding, where a draft proposes tokens and the target model checks all of
 * them in one forward pass ("Scaling TensorRT-LLM: Kernel Fusion and
 * Inflight Batching in Production", section "3. Speculative Decoding for
 * Tail Latency"; "TensorRT-LLM Guide: High-Throughput GPU Inference Engine",
 * section "2. Pipelined Speculative Decoding").  q_len >= 1 new tokens per
 * request, the same for every request of the call; new token t of request b
 * sits at position L_b + t (L_b = seq_lens[b], tokens cached before the
 * call).  Layouts: q and out [batch][q_len][Hq][d], k_new and v_new
 * [batch][q_len][Hkv][d], the rest as above.
 *
 * Step part 1 for several new tokens: each token is rotated at its position
 * and its k / v stored in slot (L_b + t) % P of page
 * block_tables[b][(L_b + t) / P], exactly as pkv_rope_append stores one new
 * token (bf16 or fp8 pools).  Positions past bt_stride * P are range errors
 * (device error word, the token is skipped). */
pkv_status pkv_rope_append_tokens(pkv_ctx* ctx, void* q, const void* k_new, const void* v_new,
                                  void* k_pool, void* v_pool,
                                  const float* k_scale, const float* v_scale,
                                  const int32_t* block_tables, int bt_stride,
                                  const int32_t* seq_lens, int batch, int q_len,
                                  cudaStream_t stream);

/* Step part 2 for several new tokens: new token t attends tokens
 * 0 .. L_b + t (the cache, the new tokens before it and itself; causal among
 * the new tokens), out[b][t][h][:] = bf16(o).  The G x q_len query rows of a
 * (request, kv head) share each K/V tile, so the cache is read once per
 * call whatever q_len is.  Needs G * q_len <= 16 (PKV_ERR_UNSUPPORTED
 * otherwise); bf16 or E4M3 pools (scales as for pkv_decode_attn, E4M3 read
 * in 16-token tiles here); requests whose L_b + q_len exceeds
 * bt_stride * P get zeros and set the device error word.  The split merge
 * runs in a second kernel, as for pkv_decode_attn. */
pkv_status pkv_decode_attn_tokens(pkv_ctx* ctx, const void* q, const void* k_pool, const void* v_pool,
                                  const float* k_scale, const float* v_scale,
                                  const int32_t* block_tables, int bt_stride,
                                  const int32_t* seq_lens, int batch, int q_len, void* out,
                                  cudaStream_t stream);

/* The whole step in one call: pkv_rope_append then pkv_decode_attn (q_len =
 * 1), or pkv_rope_append_tokens then pkv_decode_attn_tokens (q_len > 1,
 * G * q_len <= 16), with the same arguments, layouts, results and errors as
 * that pair of calls (q rotated in place, the new tokens appended, out
 * written).  The pages fuse the attention-side work of a decode step into as
 * few passes as possible ("Scaling TensorRT-LLM: Kernel Fusion and Inflight
 * Batching in Production", section "What Gets Fused"); here the attention is
 * launched as a programmatic dependent of the RoPE + append kernel, so its
 * start (the split over the SMs, the first page-table lookups) runs while
 * that kernel finishes; it reads q and issues its first tile load only once
 * the append is complete.  On a host-side error nothing is launched; if the
 * append launches and the attention does not, PKV_ERR_CUDA is returned. */
pkv_status pkv_decode_step(pkv_ctx* ctx, void* q, const void* k_new, const void* v_new,
                           void* k_pool, void* v_pool, const float* k_scale, const float* v_scale,
                           const int32_t* block_tables, int bt_stride, const int32_t* seq_lens,
                           int batch, int q_len, void* out, cudaStream_t stream);

/* Several new tokens per request, a different number for each ("varlen"):
 * chunked prefill mixed with decode in one batch ("Scaling TensorRT-LLM:
 * Kernel Fusion and Inflight Batching in Production", section "What the
 * Scheduler Actually Does"; "TensorRT-LLM Guide: High-Throughput GPU
 * Inference Engine", section "1. In-Flight Batching: Continuous Iteration
 * Scheduling").  The new tokens of all requests are packed: cu_q [batch + 1]
 * int32 on the device, cu_q[0] = 0, non-decreasing, cu_q[batch] = n_tokens;
 * token i of request b (cu_q[b] <= i < cu_q[b + 1]; a request may have none)
 * sits at position L_b + i - cu_q[b].  q [n_tokens][Hq][d], k_new / v_new
 * [n_tokens][Hkv][d], out [n_tokens][Hq][d], all bf16.
 *
 * pkv_rope_append_varlen: pkv_rope_append_tokens for packed tokens (bf16 or
 * E4M3 pools): rotates q in place, appends every new token's k / v. */
pkv_status pkv_rope_append_varlen(pkv_ctx* ctx, void* q, const void* k_new, const void* v_new,
                                  void* k_pool, void* v_pool,
                                  const float* k_scale, const float* v_scale,
                                  const int32_t* block_tables, int bt_stride,
                                  const int32_t* seq_lens, const int32_t* cu_q, int batch, int n_tokens,
                                  cudaStream_t stream);

/* pkv_decode_attn_varlen: token i of request b attends tokens 0 .. L_b + i -
 * cu_q[b] of its cache (after pkv_rope_append_varlen: the cache, the earlier
 * new tokens and itself), bf16 or E4M3 pools (scales as for
 * pkv_decode_attn).  A plan
 * kernel cuts each request's new tokens into blocks of 16 / G tokens (the G x
 * 16/G query rows of a block and kv head are one 16-row mma), each block
 * streams its prefix of the cache once for its tokens; with bf16 pools a
 * request of at least 64 / G new tokens (pkv_set_prefill_rows) is cut
 * instead into blocks of 128 / G tokens for the tensor cores (one 128-row
 * MMA block per kv head).  The context holds
 * room for 4 x max_batch blocks (at most 8192): a call with batch +
 * ceil(n_tokens / (16 / G)) above that returns PKV_ERR_UNSUPPORTED without
 * launching; lengths past the block table zero the affected tokens' output
 * and set the error word, as for pkv_decode_attn. */
pkv_status pkv_decode_attn_varlen(pkv_ctx* ctx, const void* q, const void* k_pool, const void* v_pool,
                                  const float* k_scale, const float* v_scale,
                                  const int32_t* block_tables, int bt_stride, const int32_t* seq_lens,
                                  const int32_t* cu_q, int batch, int n_tokens, void* out,
                                  cudaStream_t stream);

/* Step part 1 from the layer input: the QKV projection of the new tokens
 * fused with RoPE and the append ("Scaling TensorRT-LLM: Kernel Fusion and
 * Inflight Batching in Production", section "What Gets Fused").  x is the
 * new tokens' input [batch][hidden] bf16 (one new token per request), w_qkv
 * the projection [(Hq + 2 Hkv) d][hidden] bf16 (one row per output feature:
 * the Hq q heads, then the Hkv k heads, then the Hkv v heads; row h d + i is
 * dimension i of head h).  With y = bf16_RNE(x w_qkv^T) (fp32 accumulation on
 * the tensor cores), it does what pkv_rope_append does with q = y's q part,
 * k_new = y's k part, v_new = y's v part: q_out [batch][Hq][d] receives the
 * rotated q, rotated k and raw v go into slot L_b % P of page
 * block_tables[b][L_b / P] (bf16 or E4M3 pools).  hidden must be a multiple
 * of 64 (PKV_ERR_UNSUPPORTED otherwise); x, w_qkv and q_out 16-byte aligned.
 * Range errors as for pkv_rope_append.
 *
 * w_layout says how w_qkv is stored: PKV_W_ROWS, the row-major
 * [(Hq + 2 Hkv) d][hidden] above, or PKV_W_TILED, the same values in the
 * layout pkv_qkv_pack_weight writes, which the kernel reads as one
 * contiguous 16 KB (d = 128) run per head and 64-element slice of hidden.
 * Results are bit-identical between the two; the tiled layout is the fast
 * one (the row-major one reads 128-byte pieces 2 hidden bytes apart). */
pkv_status pkv_qkv_rope_append(pkv_ctx* ctx, const void* x, const void* w_qkv, int hidden, int w_layout,
                               void* q_out, void* k_pool, void* v_pool,
                               const float* k_scale, const float* v_scale,
                               const int32_t* block_tables, int bt_stride,
                               const int32_t* seq_lens, int batch, cudaStream_t stream);

/* Device side of the host page allocator (pkv_pages.h) for a decode loop,
 * in two small kernels on `stream`: applies the allocator's change log to a
 * device copy of the block table, then gathers the rows and lengths of the
 * step's batch into the block_tables / seq_lens arguments of the step
 * (page_size is checked to be positive; the rows are copied whole).
 *   upload    device int32 [3 n_changes + 2 batch]: the (slot, index, value)
 *             triples of pkv_pages_take_changes (each entry at most once),
 *             then the batch's slots, then their lengths L (tokens cached
 *             before the step) -- one host-to-device copy per step;
 *   table     device int32 [max_batch][max_blocks], updated in place;
 *   bt_out    device int32 [batch][max_blocks]: row b receives row slot_b
 *             of the updated table (-1 everywhere for a slot outside it);
 *   lens_out  device int32 [batch]: the lengths.
 * Triples outside the table are skipped.  All pointers 4-byte
 * aligned and caller-owned.  Asynchronous; PKV_ERR_INVALID_ARG for bad sizes
 * or pointers, PKV_ERR_CUDA on a launch failure. */
pkv_status pkv_table_sync(const int32_t* upload, int n_changes, int batch, int max_batch, int max_blocks,
                          int page_size, int32_t* table, int32_t* bt_out, int32_t* lens_out,
                          cudaStream_t stream);

/* Layouts of the QKV weight for pkv_qkv_rope_append. */
enum { PKV_W_ROWS = 0, PKV_W_TILED = 1 };

/* Writes w_qkv [(Hq + 2 Hkv) d][hidden] bf16 (row-major, as for
 * pkv_qkv_rope_append) into w_tiled in the tiled layout
 * [Hq + 2 Hkv][hidden / 64][d][64]: element (h, kb, i, j) is row h d + i,
 * column 64 kb + j of w_qkv.  A load-time step for a static weight; the
 * output has the input's size, must not overlap it, and both are 16-byte
 * aligned.  hidden a multiple of 64 (PKV_ERR_UNSUPPORTED otherwise).
 * Asynchronous on `stream`. */
pkv_status pkv_qkv_pack_weight(pkv_ctx* ctx, const void* w_qkv, int hidden, void* w_tiled,
                               cudaStream_t stream);

/* Frees the workspace.  NULL is accepted.  Synchronises the device. */
pkv_status pkv_destroy(pkv_ctx* ctx);

/* Static text for a status code. */
const char* pkv_status_str(pkv_status s);

/* Synchronises `stream`, reads and clears the context's device error word.
 * Returns PKV_OK, PKV_ERR_DEVICE_BOUNDS or PKV_ERR_DEVICE_TIMEOUT; if
 * `bits` is not NULL it receives the raw word (1: length out of range,
 * 2: page id out of range, 4: wait timed out). */
pkv_status pkv_check_device_error(pkv_ctx* ctx, cudaStream_t stream, int* bits);

/* Caps the number of warp workers pkv_decode_attn splits the token ranges
 * over (0 restores the automatic choice).  Results do not depend on it
 * beyond rounding; tests use it to force 1, 2, 7, ... splits. */
pkv_status pkv_set_workers(pkv_ctx* ctx, int workers);

/* Caps the number of dynamic chunks each warp range's tail is cut into
 * (0 .. 8; 0 gives a static split; -1, the default, is automatic: 4 chunks
 * when every range holds at least 192 tiles, as long contexts do, else a
 * static split).  With a cap above 0 the last quarter of every range (at
 * most 48 tiles of 16 tokens) is cut into chunks of at least 4 tiles that
 * warps which finish their own share early claim; ranges under 32 tiles get
 * no tail.  Results do not depend on it beyond rounding, and each chunk's
 * partial has a fixed slot, so they repeat bit for bit. */
pkv_status pkv_set_tail_chunks(pkv_ctx* ctx, int max_chunks);

/* Which requests of a pkv_decode_attn_varlen call (bf16 pools) take the
 * tensor-core prefill-chunk path: those with G x new tokens >= rows (1 ..
 * 128; 64, the default, is half a block); 0 sends every request to the
 * several-new-tokens kernel.  That path cuts a request's new tokens into
 * blocks of 128 / G, whose 128 query rows (G heads of each token) share one
 * pass over the request's cache per kv head: S = q K^T and P V on tcgen05
 * with fp32 accumulators in tensor memory, P carried as two bf16 terms
 * (about 16 significant bits).  Results agree with the other path within
 * rounding. */
pkv_status pkv_set_prefill_rows(pkv_ctx* ctx, int rows);

/* Sets how many CTAs (one thread-block cluster) share each head's hidden
 * dimension in pkv_qkv_rope_append: 1 .. 4, or 0 (the default) for the
 * automatic choice (as many as the SMs hold in one wave).  At most one
 * 64-element block of hidden per CTA.  Results do not depend on it beyond
 * the order of the fp32 sums; tests use it to cover every split. */
pkv_status pkv_set_qkv_split(pkv_ctx* ctx, int split);

/* The launch shape pkv_qkv_rope_append uses for (batch, hidden) under the
 * current split setting: shape[0] = CTAs per cluster (the split), shape[1] =
 * TMA ring stages, shape[2] = dynamic shared memory bytes per CTA, shape[3]
 * = clusters of that shape the GPU holds at once (0 if unknown; the grid has
 * (Hq + 2 Hkv) x ceil(batch / 128) clusters).  Host-only query. */
pkv_status pkv_qkv_launch_shape(pkv_ctx* ctx, int batch, int hidden, int* shape);

/* Bytes of device workspace the context holds. */
size_t pkv_workspace_bytes(const pkv_ctx* ctx);

/* pkv_decode_attn for callers that cannot allocate device memory.  The pages
 * describe no such entry point; it exists for callers such as a serving
 * runtime that reserved all device memory for its own pool at start-up, a
 * plug-in that may only use memory its host framework hands it, or a
 * latency-critical path that must not pay for an allocation and the device
 * synchronisation that can come with it.  pkv_create allocates a workspace;
 * this call allocates nothing (no cudaMalloc, cudaFree or allocating library
 * routine) and takes the shapes from cfg instead of a context.  Arguments,
 * layouts and results are those of pkv_decode_attn.
 *
 * Its scratch is one fixed device array of 16 MiB inside the library, which
 * every GPU that loads the library holds until the process exits.  A call
 * whose scratch would not fit (error word + batch + 8 ints of split geometry
 * + split partials for 8 warps per SM: 9.9 MB on a 148-SM B200 at d = 128)
 * returns PKV_ERR_UNSUPPORTED without launching.
 * The first call on a device, made with that device current, looks up the
 * array's device address and caches it; make that first call before any
 * stream capture.  Every call shares the array and the previous call's
 * contents stay in it: each call clears the part that must start at zero with
 * cudaMemsetAsync on `stream`, so calls ordered on one stream are
 * independent, but calls that overlap on the GPU race.  Device-side range
 * errors are handled as in pkv_decode_attn but cannot be read back (there is
 * no context). */
pkv_status pkv_decode_attn_noalloc(const pkv_config* cfg, const void* q, const void* k_pool,
                                   const void* v_pool, const float* k_scale, const float* v_scale,
                                   const int32_t* block_tables, int bt_stride,
                                   const int32_t* seq_lens, int batch, void* out,
                                   cudaStream_t stream);

#ifdef __cplusplus
}
#endif
#endif
