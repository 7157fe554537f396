/*
 * pagedattn.h -- C ABI of libpagedattn.so, the paged-KV attention hot path of a
 * nano-vLLM-style serving engine, for NVIDIA B200 (sm_100a).
 *
 * What the pages fix.  "Deep into the Nano-vLLM inference engine" (lnwmold.com
 * news item), section "Control plane vs. data plane": the block manager is a
 * CPU-side control plane that only tracks metadata, while the KV cache itself
 * lives on the GPU (the data plane); freed blocks are marked free and their GPU
 * memory is not cleared.  "Nano-vLLM engine architecture" (intelliparadigm.com)
 * section 3.2: GPU memory is cut into fixed-size blocks (default 256 tokens).
 * The same lnwmold.com item, section "Preparation before computation": a
 * prefill batches sequences by cumulative sequence lengths; a decode batches
 * one new token per sequence.  This library is that data plane.
 *
 * Layouts (readings; the pages defer the physical layout, section "What's
 * Next" of the lnwmold.com item):
 *   K pool, V pool   [num_blocks, block_size, num_kv_heads, head_dim]  bf16
 *                    slot s = flat token row s of [num_blocks*block_size, Hkv, D]
 *   key / value      [N, num_kv_heads, head_dim] bf16, rows key_token_stride apart
 *   q (decode)       [num_seqs, num_q_heads, head_dim] bf16, rows q_token_stride apart
 *   q (prefill)      [total_q, num_q_heads, head_dim] bf16, rows q_token_stride apart
 *   out              [rows, num_q_heads, head_dim] bf16, contiguous
 *   block_tables     [num_seqs, max_blocks_per_seq] int32 (unused entries: any value)
 *   GQA              query head h reads KV head h / (num_q_heads / num_kv_heads)
 *
 * Ownership.  The caller allocates and owns every buffer (including the decode
 * workspace).  The library never allocates, frees or synchronises; all work is
 * enqueued on `stream` (a cudaStream_t; NULL = the legacy default stream) and
 * the buffers must stay alive until it has run.  Pointers are device pointers
 * to 16-byte aligned memory; head_dim is innermost and contiguous.
 *
 * Errors.  Host-side validation runs before any launch and returns a status;
 * pa_last_error_message() gives the reason (thread-local).  A launch failure
 * returns PA_ERR_CUDA.  Device-side metadata checks: with a non-NULL err_flag
 * (device int32), kernels OR a PA_FLAG_* bit into it when metadata is out of
 * range and skip or neutralise the offending access; they never trap.  With a
 * NULL err_flag the same guards still keep every access inside the buffers
 * (out-of-range block ids read zeros), but nothing is reported.  Every wait in
 * the kernels is bounded: a wait that gives up (about two seconds) sets
 * PA_FLAG_TIMEOUT (in err_flag, and in a device-global word read by
 * pa_watchdog_read) and the kernel returns.
 *
 * Threading: the entry points are re-entrant; a per-(pointer, shape) cache of
 * TMA tensor maps is guarded by a mutex.
 */
#ifndef PAGEDATTN_H
#define PAGEDATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  PA_OK = 0,
  PA_ERR_INVALID_ARG = 1,   /* a size, pointer or alignment is invalid             */
  PA_ERR_UNSUPPORTED = 2,   /* valid, but outside what the kernels implement        */
  PA_ERR_WORKSPACE = 3,     /* decode workspace missing or smaller than required    */
  PA_ERR_CUDA = 4           /* a CUDA runtime/driver call or a launch failed        */
} pa_status;

typedef enum { PA_BF16 = 0 } pa_dtype;

/* bits OR-ed into *err_flag (checked mode) */
#define PA_FLAG_SLOT_OOB   1  /* slot_mapping entry >= num_blocks*block_size          */
#define PA_FLAG_BLOCK_OOB  2  /* block table entry outside [0, num_blocks)            */
#define PA_FLAG_LEN_OOB    4  /* context/sequence length outside its declared bounds  */
#define PA_FLAG_TIMEOUT    8  /* a bounded wait gave up                                */
#define PA_FLAG_SLOT_MISMATCH 16  /* pa_decode_store / pa_prefill_store: a slot_mapping
                                     entry is not the block-table slot of its token  */

typedef void* pa_stream_t;

#if defined(__GNUC__)
#define PA_API __attribute__((visibility("default")))
#else
#define PA_API
#endif

/* Human-readable name of a status. Never NULL. */
PA_API const char* pa_status_string(pa_status s);

/* Detail of the last non-OK status returned on this thread ("" if none). */
PA_API const char* pa_last_error_message(void);

/* Library version string, e.g. "pagedattn 0.1 sm_100a". */
PA_API const char* pa_version(void);

/*
 * pa_store_kvcache -- scatter each step's new K/V rows into the block pool.
 *
 * For i in [0, num_tokens): if slot_mapping[i] >= 0, copies key row i to flat
 * token row slot_mapping[i] of k_cache and value row i to the same row of
 * v_cache (num_kv_heads*head_dim bf16 each, bit-exact).  A negative slot means
 * padding: nothing is written.  Source: the Block Manager hands every token a
 * place in a fixed-size block ("From Sequences to Blocks", lnwmold.com item);
 * the new token's cache is written before attention reads it ("Handling
 * resource exhaustion": room for the next token's cache).
 *   key, value           device, [num_tokens, Hkv, D], rows *_token_stride
 *                        elements apart (>= Hkv*D, multiple of 8)
 *   k_cache, v_cache     device, [num_slots, Hkv, D] (num_slots = NB*block_size)
 *   slot_mapping         device int32 [num_tokens]
 *   Hkv*D must be a multiple of 8 (16-byte rows).  num_tokens == 0 is a no-op.
 * Rows that name the same slot race (the caller's control plane never does
 * that).  Slots >= num_slots are skipped (PA_FLAG_SLOT_OOB in checked mode).
 */
PA_API pa_status pa_store_kvcache(const void* key, const void* value,
                           int64_t key_token_stride, int64_t value_token_stride,
                           void* k_cache, void* v_cache,
                           const int32_t* slot_mapping, int32_t num_tokens,
                           int32_t num_kv_heads, int32_t head_dim, int64_t num_slots,
                           pa_dtype dtype, int32_t* err_flag, pa_stream_t stream);

/*
 * pa_decode_workspace_size -- bytes of workspace pa_decode needs for these
 * sizes (0 when no sequence can be split).  partition_size 0 = automatic
 * (same rule pa_decode applies), else the explicit value passed to pa_decode.
 */
PA_API size_t pa_decode_workspace_size(int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads,
                                int32_t head_dim, int32_t max_context_len,
                                int32_t partition_size);

/*
 * pa_decode -- paged decode attention with GQA (one query token per sequence).
 *
 * For sequence i and query head h (g = h / (Hq/Hkv)):
 *   out[i,h,:] = softmax_t(scale * q[i,h,:] . K_i[t,g,:]) @ V_i[t,g,:],
 *   t = 0 .. context_lens[i]-1,
 * where row t of K_i / V_i is pool row block_tables[i][t / block_size] *
 * block_size + t % block_size.  context_lens counts the new token, whose K/V
 * must already be stored.  bf16 inputs, fp32 accumulation, bf16 output.
 * Source: decode batches one new token per sequence ("Preparation before
 * computation", "Prefill and Decode", lnwmold.com item) against the paged
 * pool (intelliparadigm.com section 3.2); the attention formula itself is not
 * written on the pages (deferred to their part 2) and is the standard
 * scaled-dot-product softmax attention.
 *
 * Long contexts are split into partitions of partition_size tokens (0 =
 * automatic; else a multiple of 64) that run in parallel; their partial
 * results go to `workspace` (>= pa_decode_workspace_size bytes, 256-byte
 * aligned, caller-owned, contents need no initialisation) and a second kernel
 * merges them.  max_context_len must bound every context_lens entry (it sizes
 * the grid).  Supported: head_dim 64 or 128, block_size a power of two in
 * [16, 1024], 1 <= Hq/Hkv.  context_lens[i] == 0 gives a zero output row
 * (PA_FLAG_LEN_OOB in checked mode).
 */
PA_API pa_status pa_decode(void* out, const void* q, int64_t q_token_stride,
                    const void* k_cache, const void* v_cache,
                    const int32_t* block_tables, int32_t max_blocks_per_seq,
                    const int32_t* context_lens, int32_t num_seqs, int32_t max_context_len,
                    int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                    int32_t block_size, int32_t num_blocks, float scale,
                    int32_t partition_size, void* workspace, size_t workspace_bytes,
                    pa_dtype dtype, int32_t* err_flag, pa_stream_t stream);

/*
 * pa_decode_store -- one decode step's store_kvcache and decode in one launch.
 *
 * Same result as pa_store_kvcache(key, value, key_token_stride,
 * value_token_stride, k_cache, v_cache, slot_mapping, num_seqs, ...) followed by
 * pa_decode(...) with the remaining arguments, when slot_mapping[i] is the pool
 * slot of sequence i's newest position context_lens[i]-1 (the decode-step
 * invariant: the slot of position p is block_tables[i][p / block_size] *
 * block_size + p % block_size, "From Sequences to Blocks", lnwmold.com item;
 * the new token's K/V are written before attention reads them, "Preparation
 * before computation", same item).  The CTA of each (sequence, KV head) that
 * reads that position writes the row first, so the store costs no launch and
 * no extra pass.  key / value: [num_seqs, Hkv, D] bf16 rows (token strides in
 * elements, multiples of 8, 16-byte aligned).  slot_mapping[i] < 0 skips the
 * store of row i; >= num_blocks*block_size is skipped with PA_FLAG_SLOT_OOB;
 * a slot that breaks the invariant sets PA_FLAG_SLOT_MISMATCH (checked mode)
 * and the result is then unspecified.  Other arguments, errors and the
 * workspace as pa_decode.
 */
PA_API pa_status pa_decode_store(void* out, const void* q, int64_t q_token_stride,
                          const void* key, const void* value, int64_t key_token_stride,
                          int64_t value_token_stride, const int32_t* slot_mapping,
                          void* k_cache, void* v_cache,
                          const int32_t* block_tables, int32_t max_blocks_per_seq,
                          const int32_t* context_lens, int32_t num_seqs, int32_t max_context_len,
                          int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                          int32_t block_size, int32_t num_blocks, float scale,
                          int32_t partition_size, void* workspace, size_t workspace_bytes,
                          pa_dtype dtype, int32_t* err_flag, pa_stream_t stream);

/*
 * pa_decode_noalloc -- pa_decode for callers that cannot allocate device memory.
 *
 * The pages have no counterpart to this entry point; it exists for library
 * users.  pa_decode needs a caller-allocated workspace for long contexts.
 * Some callers cannot allocate one: an engine that reserves all GPU memory for
 * its KV pool at start-up and must not call cudaMalloc afterwards (the call
 * can fail once the pool owns the memory, and cudaFree synchronises the
 * device), or a C host program that only receives ready-made device buffers
 * from another component and has no allocator of its own.  This entry point
 * takes the same arguments as pa_decode minus the workspace and uses a fixed
 * scratch array owned by the library instead: a static device array of
 * PA_DECODE_NOALLOC_SCRATCH_BYTES (16 MiB) that every GPU which loads the
 * library holds until the process exits.  It calls no cudaMalloc, cudaFree or
 * other allocating routine.
 *   - Sizes whose split-K workspace (pa_decode_workspace_size) exceeds the
 *     scratch are rejected with PA_ERR_WORKSPACE before any launch; a larger
 *     partition_size shrinks the need.
 *   - The first call on each device (with that device current) looks up the
 *     scratch array's device address (cudaGetSymbolAddress) and remembers it
 *     for that device's context; make that first call before any stream
 *     capture.  A context re-created later (cudaDeviceReset) is noticed by its
 *     id and the address is looked up again.
 *   - Every call shares the one array, which keeps the last call's contents
 *     (nothing in it needs to start at zero).  Calls that overlap on the GPU --
 *     on two streams at once, or from two host threads -- race on it.
 */
#define PA_DECODE_NOALLOC_SCRATCH_BYTES (16u << 20)
PA_API pa_status pa_decode_noalloc(void* out, const void* q, int64_t q_token_stride,
                                   const void* k_cache, const void* v_cache,
                                   const int32_t* block_tables, int32_t max_blocks_per_seq,
                                   const int32_t* context_lens, int32_t num_seqs,
                                   int32_t max_context_len, int32_t num_q_heads,
                                   int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                                   int32_t num_blocks, float scale, int32_t partition_size,
                                   pa_dtype dtype, int32_t* err_flag, pa_stream_t stream);

/*
 * pa_prefill_varlen -- causal prefill over prompts packed by cumulative
 * sequence lengths, reading K/V from the paged pool (prefix-cached blocks
 * included).
 *
 * Sequence i computes q_len = cu_seqlens_q[i+1]-cu_seqlens_q[i] new queries
 * and has k_len = cu_seqlens_k[i+1]-cu_seqlens_k[i] keys (k_len >= q_len);
 * the first k_len-q_len keys are a cached prefix (blocks shared through the
 * hash prefix cache, "Prefix Caching via hashing", lnwmold.com item).  Query
 * j sits at absolute position k_len-q_len+j and attends keys 0 .. that
 * position (bottom-right causal alignment):
 *   out[r,h,:] = softmax_t(scale * q[r,h,:] . K_i[t,g,:]) @ V_i[t,g,:].
 * All K/V rows -- the new tokens' included -- are read from the pool, so the
 * step's pa_store_kvcache must be enqueued first on the same stream.
 *   q          device [total_q, Hq, D], rows q_token_stride elements apart
 *   out        device [total_q, Hq, D] contiguous
 *   cu_seqlens device int32 [num_seqs+1], starting at 0
 *   max_seqlen_q / max_seqlen_k bound every q_len / k_len (they size the grid)
 * Supported: head_dim 128 (tensor-core path) or 64, block_size a power of two
 * in [16, 1024].
 */
PA_API pa_status pa_prefill_varlen(void* out, const void* q, int64_t q_token_stride,
                            const void* k_cache, const void* v_cache,
                            const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k,
                            int32_t max_seqlen_q, int32_t max_seqlen_k, int32_t total_q,
                            const int32_t* block_tables, int32_t max_blocks_per_seq,
                            int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads,
                            int32_t head_dim, int32_t block_size, int32_t num_blocks,
                            float scale, pa_dtype dtype, int32_t* err_flag, pa_stream_t stream);

/*
 * pa_prefill_store -- one prefill step's store_kvcache and prefill in one launch.
 *
 * Same pool contents and output as pa_store_kvcache(key, value,
 * key_token_stride, value_token_stride, k_cache, v_cache, slot_mapping,
 * cu_seqlens_q[num_seqs], ...) followed by pa_prefill_varlen(...) with the
 * remaining arguments, when every new token's slot follows the block table:
 * slot_mapping[cu_seqlens_q[i] + j] == block_tables[i][p / block_size] *
 * block_size + p % block_size for p = k_len-q_len+j (the Block Manager's
 * mapping, "From Sequences to Blocks", lnwmold.com item; the step's new K/V
 * are written before attention reads them, "Preparation before computation",
 * same item) and no new token's slot lies in a block that another sequence of
 * the batch reads as its cached prefix (the block manager only shares full,
 * already-written blocks).  Attention reads the new keys and values straight from key /
 * value and the cached prefix from the pool, so nothing waits for the store;
 * each new (token, KV head) row is written to the pool once, by the CTA that
 * computes that token's queries, during the same launch.  A TMA box of pool
 * rows that holds both cached and new keys (a cached length that is not a
 * multiple of min(block_size, 128)) has its new rows written before it is
 * read.
 *   key, value     device [total_q, Hkv, D] bf16, rows *_token_stride elements
 *                  apart (>= Hkv*D, multiples of 8), 16-byte aligned
 *   slot_mapping   device int32 [total_q]
 * Tokens past cu_seqlens_q[num_seqs] belong to no sequence and are not stored.
 * A slot past the pool writes nothing and sets PA_FLAG_SLOT_OOB; a slot
 * (negative included) that breaks the mapping above sets
 * PA_FLAG_SLOT_MISMATCH, and that sequence's output and the pool rows it
 * touches are then unspecified.  Other arguments, limits and errors as
 * pa_prefill_varlen.  Asynchronous on `stream`.
 */
PA_API pa_status pa_prefill_store(void* out, const void* q, int64_t q_token_stride,
                                  const void* key, const void* value, int64_t key_token_stride,
                                  int64_t value_token_stride, const int32_t* slot_mapping,
                                  void* k_cache, void* v_cache, const int32_t* cu_seqlens_q,
                                  const int32_t* cu_seqlens_k, int32_t max_seqlen_q,
                                  int32_t max_seqlen_k, int32_t total_q,
                                  const int32_t* block_tables, int32_t max_blocks_per_seq,
                                  int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads,
                                  int32_t head_dim, int32_t block_size, int32_t num_blocks,
                                  float scale, pa_dtype dtype, int32_t* err_flag,
                                  pa_stream_t stream);

/*
 * pa_watchdog_read -- copy (and clear) the device-global word where kernels
 * launched without err_flag record PA_FLAG_TIMEOUT.  Synchronous on the
 * current device.  Returns PA_ERR_CUDA if the copy fails.
 */
PA_API pa_status pa_watchdog_read(uint32_t* value);

/*
 * pa_selftest_wait_timeout -- health check of the failure detection: launches a
 * one-thread kernel whose bounded mbarrier wait nothing completes; after
 * limit_us microseconds (1 .. 2,000,000) it gives up, ORs PA_FLAG_TIMEOUT into
 * *err_flag (device int32, may be NULL) and into the watchdog word, writes the
 * nanoseconds it waited to *waited_ns (device uint64, may be NULL) and returns.
 * The context stays usable.  The library's kernels bound every wait the same
 * way (about two seconds).  Asynchronous on `stream`.
 */
PA_API pa_status pa_selftest_wait_timeout(int32_t* err_flag, uint32_t limit_us,
                                          uint64_t* waited_ns, pa_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* PAGEDATTN_H */
