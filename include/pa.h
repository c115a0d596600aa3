/*
 * pa.h — C ABI of the B200 (sm_100a) paged-attention library (libpa.so).
 *
 * PagedAttention keeps each sequence's KV cache in fixed-size physical blocks
 * of a shared pool and reaches them through a per-sequence block table that
 * maps logical block i to a physical block anywhere in GPU memory
 * ("vLLM PagedAttention Deep Dive", section "Virtual Memory Paging Analogy").
 * Attention looks the blocks up, gathers K/V from them and runs standard
 * attention, with a result identical to dense attention ("vLLM PagedAttention
 * Deep Dive", section "PagedAttention Mechanism"; "PagedAttention: KV cache as
 * virtual memory", section "Interviewer follow-ups").
 *
 * Conventions shared by every call
 * --------------------------------
 *  Layout.  key_cache and value_cache are separate pools, each a contiguous
 *    T[num_blocks][num_kv_heads][block_size][head_dim] array (T = fp16 or
 *    bf16).  A token at logical position p of sequence s lives in physical
 *    block block_tables[s][p / block_size] at offset p % block_size; its slot
 *    is physical_block * block_size + offset.
 *  GQA.  Query head h reads KV head h / (num_q_heads / num_kv_heads).
 *  Pointers.  Every pointer argument is a DEVICE pointer, 16-byte aligned,
 *    owned by the caller (the library allocates nothing and keeps no pointer
 *    after a call returns).  Tensors are contiguous and row-major as stated.
 *  Streams.  Every call is asynchronous on `stream` (a cudaStream_t; NULL is
 *    the legacy default stream).  No call synchronises, except
 *    pa_get_device_error.
 *  Errors.  Host-side argument checks return PA_ERR_INVALID_ARG (null pointer,
 *    non-positive or inconsistent size, misalignment) or PA_ERR_UNSUPPORTED
 *    (a head_dim / block_size / dtype / group combination with no compiled
 *    kernel) before anything is launched.  A failed launch returns
 *    PA_ERR_CUDA.  Data-dependent errors found on the device (a slot or
 *    physical block id outside [0, num_blocks), a sequence longer than its
 *    block table, a bounded wait that ran out) never trap: the kernel records
 *    a bit in a device error word, clamps or skips the offending access, and
 *    carries on; pa_get_device_error reads and clears that word.
 *  Block sizes 16 and 32; head_dim 64 and 128; query heads per KV head 1..16.
 */
#ifndef PA_H_
#define PA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  PA_OK = 0,
  PA_ERR_INVALID_ARG = 1,
  PA_ERR_UNSUPPORTED = 2,
  PA_ERR_WORKSPACE = 3,
  PA_ERR_OUT_OF_RANGE = 4,
  PA_ERR_CUDA = 5
} pa_status;

/* Element types.  PA_FP8_E4M3 is a cache-only type (1 byte per element; see
 * pa_reshape_and_cache_fp8 / pa_decode_fp8); pa_copy_blocks accepts all three. */
typedef enum { PA_F16 = 0, PA_BF16 = 1, PA_FP8_E4M3 = 2 } pa_dtype;

/* Bits of the device error word (pa_get_device_error). */
#define PA_DEVERR_SLOT_RANGE 0x1u    /* slot_mapping entry >= num_blocks * block_size   */
#define PA_DEVERR_BLOCK_RANGE 0x2u   /* block table / block pair id outside the pool    */
#define PA_DEVERR_SEQ_RANGE 0x4u     /* sequence longer than max_blocks_per_seq blocks  */
#define PA_DEVERR_WAIT_TIMEOUT 0x8u  /* a bounded barrier wait gave up                   */

typedef struct CUstream_st *pa_stream_t; /* same type as cudaStream_t */

/* Human-readable name of a pa_status value.  Never NULL. */
const char *pa_status_string(int status);

/* Library ABI version, (major << 16) | minor.  A library service (no
 * counterpart on the pages). */
int pa_version(void);

/*
 * pa_slot_mapping — slot of every new token (logical position -> physical slot).
 *   "vLLM PagedAttention Deep Dive", "PagedAttention Mechanism" (the block table
 *   example) and "PagedAttention: KV cache as virtual memory", "Deep dive"
 *   (tokens are appended at the end of the sequence).
 * New token t belongs to sequence s with cu_q_lens[s] <= t < cu_q_lens[s+1]
 * and sits at logical position ctx_lens[s] + (t - cu_q_lens[s]).  With
 * cu_q_lens == NULL each sequence has exactly one new token (t == s, position
 * ctx_lens[s]) and num_tokens must equal num_seqs.
 *   slot_mapping  out  int64[num_tokens]
 *   block_tables  in   int32[num_seqs][max_blocks_per_seq]
 *   cu_q_lens     in   int32[num_seqs + 1] (non-decreasing, cu_q_lens[0] = 0,
 *                      cu_q_lens[num_seqs] = num_tokens) or NULL
 *   ctx_lens      in   int32[num_seqs]
 * A position past the table (block index >= max_blocks_per_seq) yields slot -1
 * and sets PA_DEVERR_SEQ_RANGE.
 */
pa_status pa_slot_mapping(int64_t *slot_mapping, const int32_t *block_tables,
                          const int32_t *cu_q_lens, const int32_t *ctx_lens, int num_seqs,
                          int num_tokens, int max_blocks_per_seq, int block_size,
                          pa_stream_t stream);

/*
 * pa_reshape_and_cache — scatter new tokens' K and V rows into their slots.
 *   "PagedAttention: KV cache as virtual memory", "Deep dive" (the lifecycle:
 *   decode takes one more block when the last one fills) and "PagedAttention:
 *   Why Static Batching Wastes Your KV Cache", "What does PagedAttention
 *   actually do differently?" (blocks are filled on demand).
 * key_cache[slot / B][h][slot % B][:] = key[t][h][:] (same for value), a bit
 * copy.  Slot -1 skips the token.  Slots must be distinct.
 *   key, value              in      T[num_tokens][num_kv_heads][head_dim]
 *   key_cache, value_cache  in/out  T[num_blocks][num_kv_heads][block_size][head_dim]
 *   slot_mapping            in      int64[num_tokens]
 * A slot >= num_blocks * block_size is skipped and sets PA_DEVERR_SLOT_RANGE.
 */
pa_status pa_reshape_and_cache(const void *key, const void *value, void *key_cache,
                               void *value_cache, const int64_t *slot_mapping, int num_tokens,
                               int num_kv_heads, int head_dim, int block_size, int num_blocks,
                               pa_dtype dtype, pa_stream_t stream);

/*
 * pa_append — pa_slot_mapping and pa_reshape_and_cache fused into one launch.
 *   "PagedAttention: KV cache as virtual memory", "Deep dive" (new tokens go
 *   to the end of the sequence, a block being taken when the last one fills)
 *   and "vLLM PagedAttention Deep Dive", "Mechanics of Chunked Prefill"
 *   (a chunk's K/V accumulate in paged blocks).
 * Each new token's slot is computed from block_tables / cu_q_lens / ctx_lens
 * (same rule as pa_slot_mapping) and its K and V rows are written there (bit
 * copy).  slot_mapping (int64[num_tokens]) receives the slots when non-NULL.
 * Same layouts and argument meanings as the two calls it fuses; a position
 * past the table sets PA_DEVERR_SEQ_RANGE and a table entry outside the pool
 * PA_DEVERR_BLOCK_RANGE (the token is skipped, its slot reported as -1).
 */
pa_status pa_append(const void *key, const void *value, void *key_cache, void *value_cache,
                    const int32_t *block_tables, const int32_t *cu_q_lens, const int32_t *ctx_lens,
                    int64_t *slot_mapping, int num_seqs, int num_tokens, int max_blocks_per_seq,
                    int num_kv_heads, int head_dim, int block_size, int num_blocks, pa_dtype dtype,
                    pa_stream_t stream);

/*
 * pa_copy_blocks — copy-on-write duplication of whole physical blocks.
 *   "PagedAttention: Why Static Batching Wastes Your KV Cache", "How does
 *   copy-on-write eliminate duplicate prompt KV cache?" (copy just that block
 *   and remap the pointer, like fork()).
 * For each pair (src, dst): key_cache[dst] = key_cache[src] and
 * value_cache[dst] = value_cache[src] (all heads, slots and dims; bit copy).
 * dst ids must be distinct and no dst may also be a src.
 *   key_cache, value_cache  in/out  T[num_blocks][num_kv_heads][block_size][head_dim]
 *                                   (T = dtype; PA_FP8_E4M3 caches are 1 byte per element)
 *   block_pairs             in      int64[num_pairs][2] = {src, dst}
 * A pair with an id outside [0, num_blocks) is skipped and sets PA_DEVERR_BLOCK_RANGE.
 */
pa_status pa_copy_blocks(void *key_cache, void *value_cache, const int64_t *block_pairs,
                         int num_pairs, int num_kv_heads, int head_dim, int block_size,
                         int num_blocks, pa_dtype dtype, pa_stream_t stream);

/*
 * pa_swap_blocks — copy whole blocks between two pools, e.g. out to a pool in
 * host memory and back.  "PagedAttention: Why Static Batching Wastes Your KV
 * Cache", "What happens when the GPU runs out of KV blocks?" (swapping:
 * evicted blocks go to CPU RAM over PCIe and come back when the sequence is
 * rescheduled).  For each pair (src, dst): dst pool block dst = src pool
 * block src, for K and V (bit copy), all pairs in one kernel launch.
 *   dst_key_cache, dst_value_cache  out  T[dst_num_blocks][num_kv_heads][block_size][head_dim]
 *   src_key_cache, src_value_cache  in   T[src_num_blocks][num_kv_heads][block_size][head_dim]
 *   block_pairs                     in   int64[num_pairs][2] = {src, dst}, device memory
 * Either pool may be pinned host memory (cudaHostAlloc / page-locked memory,
 * which the GPU addresses through unified virtual addressing); the other is
 * device memory.  dst ids must be distinct.  A pair with an id outside its
 * pool is skipped and sets PA_DEVERR_BLOCK_RANGE.
 */
pa_status pa_swap_blocks(void *dst_key_cache, void *dst_value_cache, const void *src_key_cache,
                         const void *src_value_cache, const int64_t *block_pairs, int num_pairs,
                         int num_kv_heads, int head_dim, int block_size, int src_num_blocks,
                         int dst_num_blocks, pa_dtype dtype, pa_stream_t stream);

/*
 * pa_reshape_and_cache_fp8 — pa_reshape_and_cache into FP8 (E4M3) caches.
 *   "PagedAttention: KV cache as virtual memory", "Deep dive" and
 *   "Interviewer follow-ups" (an FP8 KV cache halves the bytes per block and
 *   raises the number of sequences that fit).  The pages fix no encoding or
 *   scaling; this library's reading: OCP E4M3 without infinities (bias 7,
 *   max 448), one fp32 scale per cache, a code standing for value * scale.
 * code = nearest E4M3 of (fp32(x) / scale) — IEEE fp32 division, ties to the
 * even code, magnitudes above 448 saturate to 448.  Slot -1 skips a token.
 *   key, value              in      T[num_tokens][num_kv_heads][head_dim], T = dtype
 *   key_cache, value_cache  in/out  uint8[num_blocks][num_kv_heads][block_size][head_dim]
 *   slot_mapping            in      int64[num_tokens]
 *   k_scale, v_scale        positive finite fp32 scales of the two caches
 * head_dim must be a multiple of 16.  Out-of-range slots: as pa_reshape_and_cache.
 */
pa_status pa_reshape_and_cache_fp8(const void *key, const void *value, uint8_t *key_cache,
                                   uint8_t *value_cache, const int64_t *slot_mapping,
                                   int num_tokens, int num_kv_heads, int head_dim,
                                   int block_size, int num_blocks, float k_scale, float v_scale,
                                   pa_dtype dtype, pa_stream_t stream);

/*
 * pa_decode_partition_tokens — the split-KV partition length pa_decode uses
 * for these sizes when called with partition_tokens == 0 (a multiple of
 * block_size).  Host-only: it launches nothing and reads only the SM count of
 * the current device (148, a B200's count, when no device is visible), so the
 * choice depends on sizes and the GPU model, never on data.  The pages do not split a
 * sequence; partitioning is this library's way to spread a decode over the
 * GPU, and the combine is exact (see pa_decode).  Returns 0 for a
 * non-positive count or size or a negative max_seq_len.
 */
int pa_decode_partition_tokens(int num_seqs, int num_kv_heads, int block_size, int max_seq_len);

/*
 * pa_decode_workspace_size — bytes of scratch pa_decode needs for its split-KV
 * partial results (a library service; the pages have no workspace).
 * Host-only (launches nothing; the automatic partition length reads the
 * current device's SM count).  partition_tokens as in pa_decode (0 =
 * automatic).  Writes 0 when no sequence can span more than one partition.
 * PA_ERR_INVALID_ARG for a null `bytes`, a negative num_seqs, max_seq_len or
 * partition_tokens, or a non-positive head count, head_dim or block_size.
 */
pa_status pa_decode_workspace_size(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                                   int block_size, int max_seq_len, int partition_tokens,
                                   size_t *bytes);

/*
 * pa_decode — one query token per sequence attending over its paged K/V.
 *   "vLLM PagedAttention Deep Dive", "PagedAttention Mechanism" (look up the
 *   physical blocks, gather K/V, standard attention) and "Chunked Prefill:
 *   Preventing Compute Starvation" (decode is memory-bandwidth bound).
 * out[s][h] = softmax(scale * q[s][h] . K_s^T) V_s over the first seq_lens[s]
 * logical tokens of sequence s, K_s / V_s gathered through block_tables[s]
 * for KV head h / G.  Long sequences are cut into partitions of
 * partition_tokens tokens (0 = automatic); each partition's unnormalised
 * softmax state goes to `workspace` and a second kernel combines them with a
 * log-sum-exp reduction in a fixed order.  The arithmetic order depends only
 * on logical positions, so the output is bit-identical under any relabelling
 * of physical blocks.  seq_lens[s] == 0 gives a zero row.
 *   out           out  T[num_seqs][num_q_heads][head_dim]
 *   query         in   T[num_seqs][num_q_heads][head_dim]
 *   key_cache, value_cache in T[num_blocks][num_kv_heads][block_size][head_dim]
 *   block_tables  in   int32[num_seqs][max_blocks_per_seq]; entries past
 *                      ceil(seq_lens[s] / block_size) are never read
 *   seq_lens      in   int32[num_seqs], each <= max_seq_len
 *   max_seq_len   host upper bound of seq_lens (sizes the launch; no sync)
 *   workspace     scratch of at least pa_decode_workspace_size bytes (may be
 *                 NULL when that size is 0); returns PA_ERR_WORKSPACE if short
 * A seq_len > max_blocks_per_seq * block_size sets PA_DEVERR_SEQ_RANGE (the
 * extra tokens are ignored); a block id outside the pool is clamped to block
 * 0 and sets PA_DEVERR_BLOCK_RANGE.
 */
pa_status pa_decode(void *out, const void *query, const void *key_cache, const void *value_cache,
                    const int32_t *block_tables, const int32_t *seq_lens, int num_seqs,
                    int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                    int num_blocks, int max_blocks_per_seq, int max_seq_len,
                    int partition_tokens, float scale, pa_dtype dtype, void *workspace,
                    size_t workspace_bytes, pa_stream_t stream);

/*
 * pa_append_decode — one decode step in one launch: pa_append of every
 * sequence's new token followed by pa_decode over the grown sequences.
 *   "PagedAttention: KV cache as virtual memory", "Deep dive" (each decode
 *   step appends one token, a new block when the last one is full) and the
 *   pa_decode passages.
 * Sequence s has ctx_lens[s] cached tokens; its new token's K/V rows
 * (new_key / new_value T[num_seqs][num_kv_heads][head_dim]) are written to
 * logical position ctx_lens[s] (slot block_tables[s][ctx / block_size] *
 * block_size + ctx % block_size, bit copies), then out = attention of
 * query[s] over the ctx_lens[s] + 1 tokens.  The writes are made by the CTAs
 * that read that block, before they read it, so no second launch is needed.
 * Output and cache contents are bit-identical to pa_append + pa_decode with
 * seq_lens = ctx_lens + 1, max_seq_len = max_ctx_len + 1 and the same
 * partition_tokens and workspace (pa_decode_workspace_size with
 * max_ctx_len + 1).  slot_mapping (int64[num_seqs], may be NULL) receives
 * the slot written, -1 when none (a block id outside the pool sets
 * PA_DEVERR_BLOCK_RANGE; a context that does not fit the table sets
 * PA_DEVERR_SEQ_RANGE and nothing is written).  fp16 / bf16 caches.
 */
pa_status pa_append_decode(void *out, const void *query, const void *new_key,
                           const void *new_value, void *key_cache, void *value_cache,
                           const int32_t *block_tables, const int32_t *ctx_lens,
                           int64_t *slot_mapping, int num_seqs, int num_q_heads,
                           int num_kv_heads, int head_dim, int block_size, int num_blocks,
                           int max_blocks_per_seq, int max_ctx_len, int partition_tokens,
                           float scale, pa_dtype dtype, void *workspace, size_t workspace_bytes,
                           pa_stream_t stream);

/*
 * pa_decode_fp8 — pa_decode over FP8 (E4M3) caches (see pa_reshape_and_cache_fp8
 * for the encoding).
 *   "PagedAttention: KV cache as virtual memory", "Interviewer follow-ups"
 *   (an FP8 KV cache halves the bytes per block; attention is unchanged).
 * Attention is computed over the values code * k_scale and
 * code * v_scale; the query and output are fp16 or bf16 (`dtype`).  The
 * products run on fp16 tensor-core MMAs with fp32 accumulation: E4M3 codes
 * are exact in fp16, the query is rounded to fp16 (exact for |q| in fp16's
 * normal range).  Same arguments, partitioning, workspace
 * (pa_decode_workspace_size with the same sizes), determinism and error
 * behaviour as pa_decode.  head_dim must be 128.
 */
pa_status pa_decode_fp8(void *out, const void *query, const uint8_t *key_cache,
                        const uint8_t *value_cache, const int32_t *block_tables,
                        const int32_t *seq_lens, int num_seqs, int num_q_heads, int num_kv_heads,
                        int head_dim, int block_size, int num_blocks, int max_blocks_per_seq,
                        int max_seq_len, int partition_tokens, float scale, float k_scale,
                        float v_scale, pa_dtype dtype, void *workspace, size_t workspace_bytes,
                        pa_stream_t stream);

/*
 * pa_decode_shared_prefix — pa_decode for a batch whose sequences all begin
 * with the same cached prefix, stored once in shared physical blocks.
 *   "PagedAttention: Why Static Batching Wastes Your KV Cache", "How does
 *   copy-on-write eliminate duplicate prompt KV cache?" (sequences share the
 *   blocks of a common prompt) and "vLLM PagedAttention Deep Dive",
 *   "PagedAttention Mechanism".  Reading those blocks once for all sharers is
 *   this library's design, not the pages'.
 * Every sequence's first prefix_len tokens (a multiple of block_size, at most
 * max_seq_len and at most each seq_lens[s]) are the K/V of the physical blocks
 * prefix_blocks[0 .. prefix_len / block_size) — the same ids that lead every
 * block_tables row; the rest of each sequence is read through block_tables as
 * in pa_decode.  The split-KV partitions that lie wholly inside the prefix are
 * computed once per group of sequences (up to 16 query columns per CTA: 16 /
 * group sequences), each shared K/V tile read once for the group; the other
 * partitions and the combine are pa_decode's.  With the same partition_tokens
 * the output is bit-identical to pa_decode (each query column's arithmetic is
 * unchanged).  When no partition lies inside the prefix, or group > 8, or the
 * caches are not head_dim 128, this is pa_decode.
 *   prefix_blocks  in  int32[prefix_len / block_size] (device memory)
 * Every other argument, the workspace (pa_decode_workspace_size with the same
 * sizes) and the error behaviour as pa_decode; a sequence shorter than a
 * shared partition sets PA_DEVERR_SEQ_RANGE.  PA_ERR_INVALID_ARG for a
 * negative prefix_len, one that is not a multiple of block_size or exceeds
 * max_seq_len, or a null prefix_blocks with prefix_len > 0.
 */
pa_status pa_decode_shared_prefix(void *out, const void *query, const void *key_cache,
                                  const void *value_cache, const int32_t *prefix_blocks,
                                  int prefix_len, const int32_t *block_tables,
                                  const int32_t *seq_lens, int num_seqs, int num_q_heads,
                                  int num_kv_heads, int head_dim, int block_size, int num_blocks,
                                  int max_blocks_per_seq, int max_seq_len, int partition_tokens,
                                  float scale, pa_dtype dtype, void *workspace,
                                  size_t workspace_bytes, pa_stream_t stream);

/*
 * pa_append_decode_fp8 — pa_append_decode over FP8 (E4M3) caches: one launch
 * writes every sequence's new token as E4M3 codes (the encoding of
 * pa_reshape_and_cache_fp8: value / scale, IEEE fp32 division, nearest code
 * with ties to even, saturation at 448) and decodes over ctx_lens + 1 tokens.
 *   "PagedAttention: KV cache as virtual memory", "Deep dive" (each decode
 *   step appends one token) and "Interviewer follow-ups" (FP8 KV cache).
 * new_key / new_value are T[num_seqs][num_kv_heads][head_dim] (T = dtype,
 * fp16 or bf16, the query's type); key_cache / value_cache hold the codes.
 * Output and cache contents are bit-identical to pa_slot_mapping +
 * pa_reshape_and_cache_fp8 + pa_decode_fp8 with seq_lens = ctx_lens + 1,
 * max_seq_len = max_ctx_len + 1 and the same partition_tokens and workspace
 * (pa_decode_workspace_size with max_ctx_len + 1).  slot_mapping (int64[num_seqs],
 * may be NULL) and the error behaviour are those of pa_append_decode.
 * head_dim must be 128.
 */
pa_status pa_append_decode_fp8(void *out, const void *query, const void *new_key,
                               const void *new_value, uint8_t *key_cache, uint8_t *value_cache,
                               const int32_t *block_tables, const int32_t *ctx_lens,
                               int64_t *slot_mapping, int num_seqs, int num_q_heads,
                               int num_kv_heads, int head_dim, int block_size, int num_blocks,
                               int max_blocks_per_seq, int max_ctx_len, int partition_tokens,
                               float scale, float k_scale, float v_scale, pa_dtype dtype,
                               void *workspace, size_t workspace_bytes, pa_stream_t stream);

/*
 * pa_decode_static_workspace — pa_decode for callers that cannot allocate
 * device memory.  (No counterpart on the pages: this is a library service,
 * not part of the paged-attention method.)
 * Some callers cannot call cudaMalloc: for example a plugin running inside an
 * inference runtime that owns and budgets all device memory itself, or a
 * latency-critical serving loop that must not allocate after start-up (an
 * allocation can synchronise the device and can fail under memory pressure).
 * This entry point takes the same arguments as pa_decode minus the
 * workspace: its split-KV scratch lives in one file-scope device array of
 * PA_STATIC_WORKSPACE_BYTES bytes that every GPU which loads the library
 * holds until the process exits.  It allocates nothing itself.
 *   - Requests whose pa_decode_workspace_size exceeds
 *     PA_STATIC_WORKSPACE_BYTES return PA_ERR_WORKSPACE before any launch.
 *   - The first call on a device (with that device current) resolves the
 *     array's device address with cudaGetSymbolAddress and caches it; make
 *     that first call before any stream capture.  The cached address lives as
 *     long as the device's primary context: do not reset the device
 *     (cudaDeviceReset) between calls, or the next call would hand the
 *     kernels a stale address.
 *   - Every call on a device shares the one array, and it keeps the last
 *     call's contents.  The decode kernels write every partial result before
 *     they read it, so nothing needs clearing; but calls that overlap on the
 *     GPU (e.g. on two streams at once) race on the array and must be
 *     serialised by the caller.
 */
#define PA_STATIC_WORKSPACE_BYTES (16u << 20)

pa_status pa_decode_static_workspace(void *out, const void *query, const void *key_cache,
                                     const void *value_cache, const int32_t *block_tables,
                                     const int32_t *seq_lens, int num_seqs, int num_q_heads,
                                     int num_kv_heads, int head_dim, int block_size,
                                     int num_blocks, int max_blocks_per_seq, int max_seq_len,
                                     int partition_tokens, float scale, pa_dtype dtype,
                                     pa_stream_t stream);

/*
 * pa_prefill_chunk — causal chunked-prefill attention against the paged context.
 *   "vLLM PagedAttention Deep Dive", "Mechanics of Chunked Prefill" (a long
 *   prompt is processed chunk by chunk; each chunk's KV accumulates in paged
 *   blocks) and "PagedAttention Mechanism".
 * Sequence s has ctx_lens[s] tokens already cached and a chunk of
 * n_s = cu_q_lens[s+1] - cu_q_lens[s] query tokens whose own K/V have already
 * been written (pa_reshape_and_cache) at positions ctx_lens[s] .. ctx_lens[s]
 * + n_s - 1.  Chunk query i (absolute position ctx_lens[s] + i) attends to
 * positions 0 .. ctx_lens[s] + i inclusive.  Runs on the tcgen05 tensor cores
 * (bf16/fp16 operands, fp32 accumulation in tensor memory).
 *   out        out  T[total_q][num_q_heads][head_dim]
 *   query      in   T[total_q][num_q_heads][head_dim]
 *   cu_q_lens  in   int32[num_seqs + 1], cu_q_lens[num_seqs] == total_q
 *   ctx_lens   in   int32[num_seqs]
 *   max_q_len, max_ctx_len  host upper bounds (size the launch; no sync)
 *   workspace  device scratch of at least pa_prefill_workspace_size bytes, or
 *              NULL.  The work is one CTA per 256 chunk rows of a query head
 *              of a sequence, one CTA per SM at a time; with a workspace, the
 *              units of the last, partly filled wave are split along the key
 *              range into 2-4 parts when that shortens the tail, and their
 *              partial results are combined in part order (deterministic; this call zeroes the
 *              workspace's counters on `stream` first).  Calls sharing a
 *              workspace must be ordered.  Without one every unit runs
 *              whole; the two differ only in fp32 rounding order.
 * head_dim 64 or 128 (else PA_ERR_UNSUPPORTED).
 */
pa_status pa_prefill_workspace_size(int head_dim, size_t *bytes);
pa_status pa_prefill_chunk(void *out, const void *query, const void *key_cache,
                           const void *value_cache, const int32_t *block_tables,
                           const int32_t *cu_q_lens, const int32_t *ctx_lens, int num_seqs,
                           int total_q, int max_q_len, int max_ctx_len, int num_q_heads,
                           int num_kv_heads, int head_dim, int block_size, int num_blocks,
                           int max_blocks_per_seq, float scale, pa_dtype dtype, void *workspace,
                           size_t workspace_bytes, pa_stream_t stream);

/*
 * pa_mixed_attention — one launch for a batch that mixes decode rows and
 * prefill chunks.  "vLLM PagedAttention Deep Dive", "Mechanics of Chunked
 * Prefill" (the scheduler batches the ongoing decode tokens together with a
 * chunk of a long prompt, so decode is not starved while the prompt is
 * processed).
 * Same rule as pa_prefill_chunk for every sequence: sequence s has
 * ctx_lens[s] tokens cached before this step and n_s = cu_q_lens[s+1] -
 * cu_q_lens[s] query rows whose K/V are already written (pa_append with
 * cu_q_lens) at positions ctx_lens[s] .. ctx_lens[s] + n_s - 1; row i sees
 * positions 0 .. ctx_lens[s] + i.
 *   Sequences 0 .. num_decode_seqs - 1 are decode rows: exactly one query
 *   each, at row s (cu_q_lens[s] == s); a decode row attends over
 *   ctx_lens[s] + 1 tokens.  Given the same partition_tokens > 0, its result
 *   is bit-identical to pa_decode with seq_lens = ctx_lens + 1 and
 *   max_seq_len = max_ctx_len + 1 (with 0, this call picks its own partition
 *   length: pa_decode's choice capped at 1024 tokens).  A decode sequence
 *   whose cu_q_lens disagree sets PA_DEVERR_SEQ_RANGE.
 *   Sequences num_decode_seqs .. num_seqs - 1 are prefill chunks (any length,
 *   0 included); their rows are bit-identical to pa_prefill_chunk without a
 *   workspace (no key-range split).
 *   out, query    T[total_q][num_q_heads][head_dim]
 *   max_q_len     host upper bound on the prefill chunks' lengths
 *   max_ctx_len   host upper bound on ctx_lens over all sequences;
 *                 max_ctx_len + 1 <= max_blocks_per_seq * block_size
 *   workspace     device scratch of at least pa_mixed_workspace_size bytes
 *                 (0 when there are no decode rows: may then be NULL): the
 *                 decode rows' work-item queue counter, which this call
 *                 zeroes on `stream` before its launch, and their split-KV
 *                 partials.  Calls sharing a workspace must be ordered.
 * One kernel launch covers both kinds of rows (plus the split-KV combine of
 * the decode rows when they span several partitions, and the 4-byte memset
 * of the queue counter); it runs as clusters of two CTAs, one TPC each.
 * head_dim must be 128; fp16 / bf16 caches; group <= 16.
 */
pa_status pa_mixed_workspace_size(int num_decode_seqs, int num_q_heads, int num_kv_heads,
                                  int head_dim, int block_size, int max_ctx_len,
                                  int partition_tokens, size_t *bytes);
pa_status pa_mixed_attention(void *out, const void *query, const void *key_cache,
                             const void *value_cache, const int32_t *block_tables,
                             const int32_t *cu_q_lens, const int32_t *ctx_lens, int num_seqs,
                             int num_decode_seqs, int total_q, int max_q_len, int max_ctx_len,
                             int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                             int num_blocks, int max_blocks_per_seq, int partition_tokens,
                             float scale, pa_dtype dtype, void *workspace,
                             size_t workspace_bytes, pa_stream_t stream);

/* ------------------------------------------------------------------------
 * Host block manager — the allocator that produces block tables, slot
 * mappings and copy-on-write pairs for the kernels above.  Host memory only;
 * no CUDA call.  "PagedAttention: KV cache as virtual memory", "Deep dive"
 * (a block pool with an O(1) free queue in eviction order, per-block
 * reference counts, a prefix cache keyed by the hash of a full block's tokens
 * and its parent's key, allocate-on-append, free at count zero) and
 * "PagedAttention: Why Static Batching Wastes Your KV Cache", "How does
 * copy-on-write eliminate duplicate prompt KV cache?" (a sequence about to
 * write into a shared block gets its own copy).  Not thread-safe: one
 * manager per scheduler thread.  Sequence ids are caller-chosen int64.
 * ------------------------------------------------------------------------ */
typedef struct pa_block_manager pa_block_manager;

/* Pool of num_blocks blocks of block_size tokens; enable_prefix_caching != 0
 * turns on full-block prefix sharing.  Blocks are handed out 0, 1, 2, ...
 * while the pool is fresh.  PA_ERR_INVALID_ARG (nothing created) for a null
 * `out`, a non-positive size, num_blocks * block_size above INT32_MAX (token
 * counts and positions are int), or when the host tables cannot be
 * allocated.  The handle is owned by the caller until pa_bm_destroy. */
pa_status pa_bm_create(int num_blocks, int block_size, int enable_prefix_caching,
                       pa_block_manager **out);
void pa_bm_destroy(pa_block_manager *bm);

/* Admit a sequence with its prompt tokens (tokens[num_tokens], host memory,
 * read during the call only): leading full blocks whose prefix key is cached
 * are shared (reference count + 1, revived from the free queue if needed);
 * the rest come from the front of the free queue.  Writes the number of
 * prompt tokens whose K/V are already cached (num_cached_tokens may be NULL).
 * PA_ERR_INVALID_ARG for an id already in use, a negative count or a null
 * `tokens` with num_tokens > 0; PA_ERR_OUT_OF_RANGE when the pool cannot hold
 * the prompt.  State is unchanged on every error. */
pa_status pa_bm_add_sequence(pa_block_manager *bm, int64_t seq_id, const int32_t *tokens,
                             int num_tokens, int *num_cached_tokens);

/* Append generated tokens.  A new block is taken whenever the last one is
 * full.  If the last block is partially filled and shared (count > 1), it is
 * first replaced by a fresh block and the (src, dst) pair is queued for
 * pa_bm_take_copies (copy-on-write).  PA_ERR_INVALID_ARG for an unknown id, a
 * negative count or a null `tokens` with num_tokens > 0; PA_ERR_OUT_OF_RANGE
 * when the pool runs out.  State is unchanged on every error. */
pa_status pa_bm_append(pa_block_manager *bm, int64_t seq_id, const int32_t *tokens,
                       int num_tokens);

/* The child shares every block of the parent (parallel sampling, beam search).
 * PA_ERR_INVALID_ARG (state unchanged) for an unknown parent or a child id
 * already in use. */
pa_status pa_bm_fork(pa_block_manager *bm, int64_t parent_id, int64_t child_id);

/* Finish a sequence: every block's count drops by one; blocks reaching zero
 * go to the back of the free queue, last logical block first.  Cached full
 * blocks keep their key until reused, so later prompts can still hit them.
 * PA_ERR_INVALID_ARG for an unknown id. */
pa_status pa_bm_free(pa_block_manager *bm, int64_t seq_id);

/* The sequence's physical blocks in logical order into out[capacity] (host
 * memory; the rest filled with -1).  *num_blocks (may be NULL) gets the
 * table's length even when capacity is too small, which returns
 * PA_ERR_WORKSPACE and writes nothing to `out`.  PA_ERR_INVALID_ARG for an
 * unknown id, a negative capacity or a null `out` with capacity > 0. */
pa_status pa_bm_block_table(const pa_block_manager *bm, int64_t seq_id, int32_t *out,
                            int capacity, int *num_blocks);

/* Slots of logical positions start .. start + count - 1 (physical * B + offset)
 * into out[count] (host memory).  Positions may run past the tokens held, up
 * to the end of the sequence's last block; beyond it PA_ERR_OUT_OF_RANGE and
 * nothing is written.  PA_ERR_INVALID_ARG for an unknown id, a negative start
 * or count, or a null `out` with count > 0. */
pa_status pa_bm_slots(const pa_block_manager *bm, int64_t seq_id, int start, int count,
                      int64_t *out);

/* Move the queued copy-on-write pairs into pairs[capacity][2] (host memory,
 * (src, dst) in queue order) and return how many; returns minus the number
 * pending (and takes none) if capacity is too small, and -1 for a null
 * manager, a negative capacity or a null `pairs` with capacity > 0. */
int pa_bm_take_copies(pa_block_manager *bm, int64_t *pairs, int capacity);

/* Counters; each returns -1 for a null manager, an out-of-range block or an
 * unknown sequence id. */
int pa_bm_num_free_blocks(const pa_block_manager *bm);
int pa_bm_ref_count(const pa_block_manager *bm, int block);
int pa_bm_num_tokens(const pa_block_manager *bm, int64_t seq_id);

/*
 * pa_selftest_wait_timeout — a library service (no counterpart on the
 * pages): exercises the bounded-wait failure path on the GPU without
 * breaking anything.  One CTA of two roles waits on barriers that nothing
 * arrives on: role 0 gives up after limit_ns nanoseconds and raises the
 * CTA's abort word; role 1, which has the kernels' normal 4 s limit, sees the
 * word and gives up right after.  PA_DEVERR_WAIT_TIMEOUT is then set in the
 * device error word (read it with pa_get_device_error) and the context stays
 * usable.  Every kernel of this library handles a lost arrival the same way:
 * the first wait that runs out ends the whole CTA.
 *   limit_ns   1,000 .. 100,000,000 (1 us .. 100 ms), else PA_ERR_INVALID_ARG
 *   waited_ns  out  uint64[2] device memory (8-byte aligned) receiving each
 *              role's waiting time in ns, or NULL
 */
pa_status pa_selftest_wait_timeout(uint64_t limit_ns, uint64_t *waited_ns, pa_stream_t stream);

/*
 * pa_get_device_error — a library service (no counterpart on the pages):
 * synchronise `stream`, then read and clear the device error word of the
 * current device (a bitwise OR of PA_DEVERR_* since the last read).  Returns
 * PA_ERR_OUT_OF_RANGE when the word was non-zero, PA_ERR_CUDA if the
 * synchronisation or the copies fail.  The read and the clear are two copies:
 * a kernel still running on another stream can set a bit between them and
 * that bit is lost, so synchronise every stream that launched library
 * kernels before calling this.
 */
pa_status pa_get_device_error(unsigned int *error_word, pa_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* PA_H_ */
