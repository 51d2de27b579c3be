/*
 * pagedkv.h - C ABI of libpagedkv.so: paged single-query decode attention and
 * the two kernels that maintain a paged KV cache, for NVIDIA B200 (sm_100a).
 *
 * What the operations are (sources cited by page title and section):
 *
 *  - The KV cache of a sequence is cut into fixed-size blocks of B tokens that
 *    live anywhere in one shared physical pool; a per-sequence block table maps
 *    logical block j to its physical block.  Attention follows the table,
 *    gathers the scattered blocks and computes softmax(Q K^T) V.
 *    ("PagedAttention - Efficient Memory Management for LLM Serving with vLLM",
 *    section "Method (PagedAttention + vLLM)"; "LLM Inference 8 - PagedAttention",
 *    section "PagedAttention", block-table example 0->4, 1->1, 2->7.)
 *  - Each new token's K and V are stored into the cache and reused by later
 *    steps; a new block is taken only when the current one is full.
 *    ("LLM Inference 8 - PagedAttention", sections "KV Cache의 메모리 문제" and
 *    "PagedAttention의 동작 방식".)
 *  - Sequences that share a prefix share its physical blocks; when one of them
 *    writes, only that block is copied (copy-on-write, P3 -> P9 in the
 *    framework-overview flowchart of the paper digest's "방법 (Method)" section).
 *
 * Layout (the pages fix only the logical->physical indirection; this is the
 * library's choice): K and V are separate pools, each [num_blocks][num_heads]
 * [block_size][head_dim], row-major, in one storage dtype.  Token t of sequence
 * s, head h is element (block_tables[s][t / B], h, t % B, :).  One (block, head)
 * chunk is B * head_dim contiguous elements.
 *
 * Conventions for every entry point:
 *  - All data pointers are DEVICE pointers owned by the caller; the library keeps
 *    no reference after the call returns.
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *    stream) and never synchronise the host, except pkv_get_device_error.
 *  - Return 0 (PKV_OK) or a negative PKV_E* code.  Argument checks happen on the
 *    host before any CUDA call; a rejected call launches nothing and touches no
 *    memory.
 *  - Device-side checks (block id outside [0, num_blocks), context length outside
 *    [0, max_blocks_per_seq * B], slot outside [-1, num_blocks * B), copy pair
 *    outside the pool, a bounded wait that ran out) skip the offending access
 *    and set a sticky per-device error word; no kernel traps.  Outputs that
 *    depend on a flagged access are unspecified.  Read the word with
 *    pkv_get_device_error.
 *  - Supported: head_dim in {64, 128}; block_size in {8, 16, 32, 64, 128};
 *    storage dtype fp32, fp16 or bf16.  q, K, V, new K/V, out and workspace
 *    pointers must be 16-byte aligned.
 */
#ifndef PAGEDKV_H_
#define PAGEDKV_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Storage dtype of q, the K/V pools and appended rows. */
typedef enum { PKV_F32 = 0, PKV_F16 = 1, PKV_BF16 = 2 } pkv_dtype;

/* Return codes. */
enum {
  PKV_OK = 0,
  PKV_EINVAL = -1,        /* a null pointer, a negative or too-large size, bad partition size;
                             attention calls also reject num_seqs > 65535, (query tokens x) query
                             heads > 65535 and more than 32767 partitions per sequence (a work
                             unit packs the sequence and partition indices into 16 bits each) */
  PKV_EDTYPE = -2,        /* dtype is not a pkv_dtype */
  PKV_EALIGN = -3,        /* a pointer is not aligned as required */
  PKV_EUNSUPPORTED = -4,  /* head_dim or block_size not in the supported set */
  PKV_ECUDA = -5,         /* a CUDA runtime call or a kernel launch failed */
  PKV_EWORKSPACE = -6,    /* workspace smaller than paged_attn_decode_workspace_size() */
  PKV_EDEVICE = -7,       /* a kernel flagged bad device data (see pkv_get_device_error) */
  PKV_ETIMEOUT = -8,      /* a kernel's bounded wait ran out (see pkv_get_device_error) */
  PKV_ENOMEM = -9,        /* block manager: not enough free blocks (nothing was changed) */
  PKV_ESEQ = -10,         /* block manager: unknown sequence, sequence exists, or repeated in a batch */
  PKV_EOVERLAP = -11      /* debug checks: copy pairs overlap, or two appended tokens share a slot */
};

/* Reasons stored in the device error word (the `reason` of pkv_get_device_error). */
enum {
  PKV_DEV_OK = 0,
  PKV_DEV_BLOCK_ID = 1,     /* a block-table entry outside [0, num_blocks) was needed */
  PKV_DEV_CONTEXT_LEN = 2,  /* a context length outside [0, max_blocks_per_seq * B] */
  PKV_DEV_SLOT = 3,         /* an append slot >= num_blocks * B */
  PKV_DEV_COPY_PAIR = 4,    /* a copy pair with a block id outside [0, num_blocks) */
  PKV_DEV_WAIT_TIMEOUT = 5  /* a shared-memory pipeline wait exceeded its bound */
};

/*
 * paged_attn_decode - one query token per sequence attends over its paged context.
 *
 * For every sequence s < num_seqs and head h < num_heads:
 *   out[s][h][:] = sum_t w_t * V_t,  w = softmax_t(scale * <q[s][h], K_t>),
 * over the context_lens[s] tokens t reached through block_tables[s]
 * ("PagedAttention - Efficient Memory Management for LLM Serving with vLLM",
 * section "Method (PagedAttention + vLLM)").  A context of length 0 gives out = 0.
 *
 *   q             [num_seqs][num_heads][head_dim], storage dtype.
 *   k_cache,
 *   v_cache       [num_blocks][num_heads][block_size][head_dim], storage dtype.
 *   block_tables  int32 [num_seqs][max_blocks_per_seq]; entries past a sequence's
 *                 last block are never read (pad with -1).
 *   context_lens  int32 [num_seqs], 0 <= ctx <= max_blocks_per_seq * block_size.
 *   scale         multiplies q.k before the softmax (typically 1/sqrt(head_dim)).
 *   out           float32 [num_seqs][num_heads][head_dim].
 *   partition_tokens  split-context partition size in tokens: 0 = library choice
 *                 (no split when there are >= 1184 (sequence, head) pairs and
 *                 max_blocks_per_seq * block_size <= 4096, or when that maximum is
 *                 <= 512; otherwise 512); else a positive multiple of block_size.
 *                 A context longer than one partition is processed as independent
 *                 partitions whose partial softmax states are merged exactly
 *                 (log-sum-exp); a partition size >= max_blocks_per_seq *
 *                 block_size means no split.
 *   workspace     device scratch of at least paged_attn_decode_workspace_size()
 *                 bytes, 16-byte aligned.  It holds the call's work list (a few
 *                 bytes per sequence) and, when the call splits, the partitions'
 *                 partial softmax states.  Contents on entry do not matter; calls
 *                 that share one workspace must be ordered on one stream.  If NULL,
 *                 the library takes it from the stream-ordered allocator
 *                 (cudaMallocAsync / cudaFreeAsync on `stream`).
 *   stream        cudaStream_t.
 */
int paged_attn_decode(const void* q, const void* k_cache, const void* v_cache,
                      const int32_t* block_tables, const int32_t* context_lens,
                      int num_seqs, int num_heads, int head_dim, int block_size,
                      int max_blocks_per_seq, int num_blocks, pkv_dtype dtype,
                      float scale, float* out, int partition_tokens,
                      void* workspace, size_t workspace_bytes, void* stream);

/*
 * Workspace bytes paged_attn_decode needs for these sizes and partition_tokens
 * (0 = the library's choice, resolved exactly as paged_attn_decode resolves it):
 * 16 + 8 * num_seqs * P rounded up to 16, plus 8 * S * H * P and
 * 4 * S * H * P * head_dim (each rounded up to 16) when the call splits into
 * P > 1 partitions.
 * Returns (size_t)-1 for arguments paged_attn_decode would reject.  Pure host
 * function.
 */
size_t paged_attn_decode_workspace_size(int num_seqs, int num_heads, int head_dim,
                                        int block_size, int max_blocks_per_seq,
                                        int partition_tokens);

/*
 * The partition size paged_attn_decode will use for these arguments (resolving
 * partition_tokens = 0), or a negative PKV_E* code.  Pure host function.
 */
int paged_attn_decode_partition_tokens(int num_seqs, int num_heads, int head_dim,
                                       int block_size, int max_blocks_per_seq,
                                       int partition_tokens);

/*
 * paged_attn_decode_gqa - paged_attn_decode for grouped-query attention.
 *
 * num_heads query heads share num_kv_heads K/V heads (num_heads a multiple of
 * num_kv_heads): query head h reads K/V head h / (num_heads / num_kv_heads).  The
 * digest ("PagedAttention - Efficient Memory Management for LLM Serving with
 * vLLM", related work) names fewer K/V heads (GQA) as a way to shrink the KV cache
 * that is orthogonal to paging.
 *
 *   q, out        [num_seqs][num_heads][head_dim] (q in the storage dtype, out fp32).
 *   k_cache,
 *   v_cache       [num_blocks][num_kv_heads][block_size][head_dim].
 *   Every other argument, the return codes and the device-side checks are those of
 *   paged_attn_decode; num_kv_heads == num_heads is exactly paged_attn_decode.
 *   The workspace size comes from paged_attn_decode_gqa_workspace_size.
 *
 * With 16-bit K/V, 2 <= G <= 16 query heads per K/V head run on a warp-level
 * tensor-core kernel (16-row tiles) and 16 < G <= 128 on a tcgen05 kernel (one
 * 128-row tile per (sequence, K/V head)); fp32 K/V and other G on CUDA cores.
 */
int paged_attn_decode_gqa(const void* q, const void* k_cache, const void* v_cache,
                          const int32_t* block_tables, const int32_t* context_lens,
                          int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                          int block_size, int max_blocks_per_seq, int num_blocks,
                          pkv_dtype dtype, float scale, float* out, int partition_tokens,
                          void* workspace, size_t workspace_bytes, void* stream);

/* Workspace bytes paged_attn_decode_gqa needs; (size_t)-1 for rejected arguments. */
size_t paged_attn_decode_gqa_workspace_size(int num_seqs, int num_heads, int num_kv_heads,
                                            int head_dim, int block_size,
                                            int max_blocks_per_seq, int partition_tokens);

/* Partition size paged_attn_decode_gqa will use (the library's choice counts
 * (sequence, K/V head) pairs), or a negative PKV_E* code.  Pure host function. */
int paged_attn_decode_gqa_partition_tokens(int num_seqs, int num_heads, int num_kv_heads,
                                           int head_dim, int block_size,
                                           int max_blocks_per_seq, int partition_tokens);

/*
 * paged_attn_decode_tune - choose the split-context partition size for these inputs
 * by measurement (the digest's discussion asks whether block size should be tuned per
 * model and workload rather than hard-coded; the partition size is the part that can
 * be changed per call).
 *
 * Runs paged_attn_decode_gqa on the given inputs for each candidate partition size
 * (no split, then 4096, 2048, ... 64 tokens that are multiples of block_size and
 * shorter than the longest possible context): one untimed call and `reps` timed
 * calls each, timed with CUDA events on `stream`.  Synchronises the stream.  Returns
 * the fastest partition size (> 0) or a negative PKV_E* code; `out` ends up holding
 * the decode result for the chosen size.  times_ms / candidates (may be NULL, up to
 * max_candidates entries) receive the mean time per call and the candidate sizes;
 * *num_candidates (may be NULL) the number of candidates (at most 8).
 *
 *   workspace     at least paged_attn_decode_tune_workspace_size() bytes (required).
 *   Other arguments as in paged_attn_decode_gqa.
 */
int paged_attn_decode_tune(const void* q, const void* k_cache, const void* v_cache,
                           const int32_t* block_tables, const int32_t* context_lens,
                           int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                           int block_size, int max_blocks_per_seq, int num_blocks,
                           pkv_dtype dtype, float scale, float* out, void* workspace,
                           size_t workspace_bytes, int reps, float* times_ms, int* candidates,
                           int max_candidates, int* num_candidates, void* stream);

/* Workspace bytes paged_attn_decode_tune needs (the largest over its candidates). */
size_t paged_attn_decode_tune_workspace_size(int num_seqs, int num_heads, int num_kv_heads,
                                             int head_dim, int block_size,
                                             int max_blocks_per_seq);

/*
 * paged_attn_multi_query - several query tokens per sequence over its paged context.
 *
 * For a prefill chunk appended to a cached prefix, or draft tokens checked in one
 * pass (the video summary "KV 캐시·PagedAttention로 LLM 추론 속도와 GPU 처리량 높이기",
 * "주요 인사이트": chunked prefill, speculative decoding).  The q_len new tokens are
 * already in the cache as the last q_len of the context_lens[s] tokens; query token
 * j (0-based) of sequence s attends the first context_lens[s] - q_len + j + 1
 * tokens (causal), or none when that count is not positive (its row is zero).
 * num_heads query heads share num_kv_heads K/V heads as in paged_attn_decode_gqa.
 *
 *   q             [num_seqs][q_len][num_heads][head_dim], fp16 or bf16.
 *   out           float32 [num_seqs][q_len][num_heads][head_dim].
 *   The rest is as in paged_attn_decode_gqa; fp32 storage returns PKV_EUNSUPPORTED.
 *   q_len = 1 computes exactly what paged_attn_decode_gqa computes.
 *
 * R = q_len * G query rows per (sequence, K/V head): R <= 16 runs on the warp-level
 * tensor-core kernel; R > 16 (with G <= 128 and head_dim 64 or 128) on the tcgen05
 * kernel, 128-row tiles of floor(128 / G) query tokens, K/V read once per tile.
 */
int paged_attn_multi_query(const void* q, const void* k_cache, const void* v_cache,
                           const int32_t* block_tables, const int32_t* context_lens,
                           int num_seqs, int q_len, int num_heads, int num_kv_heads,
                           int head_dim, int block_size, int max_blocks_per_seq, int num_blocks,
                           pkv_dtype dtype, float scale, float* out, int partition_tokens,
                           void* workspace, size_t workspace_bytes, void* stream);

/* Workspace bytes paged_attn_multi_query needs; (size_t)-1 for rejected arguments. */
size_t paged_attn_multi_query_workspace_size(int num_seqs, int q_len, int num_heads,
                                             int num_kv_heads, int head_dim, int block_size,
                                             int max_blocks_per_seq, int partition_tokens);

/*
 * kv_cache_append - store the step's new K and V rows into their cache slots.
 *
 * For every token t < num_tokens with slot = slot_mapping[t] >= 0:
 *   k_cache[slot / B][h][slot % B][:] = k[t][h][:]   (and the same for v), all h.
 * ("LLM Inference 8 - PagedAttention", section "KV Cache의 메모리 문제": the new
 * token's Key and Value are added to the cache.)  slot = -1 skips the token; a
 * slot >= num_blocks * B is skipped and flagged (PKV_DEV_SLOT).  Two tokens
 * with the same slot race (unspecified which one lands) unless debug checks are
 * on (pkv_set_debug_checks): then the call copies slot_mapping to the host,
 * synchronising the stream, and returns PKV_EOVERLAP without launching when
 * pkv_check_slots rejects it.  Bit-exact copy.
 *
 *   k, v          [num_tokens][num_heads][head_dim], storage dtype.
 *   slot_mapping  int64 [num_tokens].
 */
int kv_cache_append(const void* k, const void* v, void* k_cache, void* v_cache,
                    const int64_t* slot_mapping, int num_tokens, int num_heads,
                    int head_dim, int block_size, int num_blocks, pkv_dtype dtype,
                    void* stream);

/*
 * kv_block_copy - copy-on-write block copies.
 *
 * For every pair i < num_pairs, (src, dst) = (src_dst_pairs[2i], src_dst_pairs[2i+1]):
 *   k_cache[dst] = k_cache[src] and v_cache[dst] = v_cache[src]
 * (all heads, all block_size slots).  ("PagedAttention - Efficient Memory
 * Management for LLM Serving with vLLM", section "Method (PagedAttention +
 * vLLM)", copy-on-write: only the written block is copied.)  Pairs must not
 * overlap: no dst may repeat or appear as any src, and src != dst (a copy always
 * fills a fresh block, as in the digest's flowchart: P3 -> P9); one src may feed
 * several dsts.  Overlapping pairs race unless debug checks are on
 * (pkv_set_debug_checks): then the call copies the pairs to the host,
 * synchronising the stream, and returns PKV_EOVERLAP without launching when
 * pkv_check_copy_pairs rejects them.  A pair with an id outside [0, num_blocks)
 * is skipped and flagged (PKV_DEV_COPY_PAIR).  Bit-exact copy.
 *
 *   src_dst_pairs int64 [num_pairs][2], device memory.
 */
int kv_block_copy(void* k_cache, void* v_cache, const int64_t* src_dst_pairs,
                  int num_pairs, int num_heads, int head_dim, int block_size,
                  int num_blocks, pkv_dtype dtype, void* stream);

/*
 * Overlap checks of the cache-maintenance inputs, on host arrays (no CUDA call).
 *
 * pkv_check_copy_pairs: PKV_EOVERLAP if some pair has src == dst, some dst
 *   appears twice, or some dst is also a src; else PKV_OK.  Pairs with a
 *   negative id copy nothing and are ignored.  host_pairs is int64
 *   [num_pairs][2] (src, dst) in host memory.
 * pkv_check_slots: PKV_EOVERLAP if two tokens have the same slot >= 0; else
 *   PKV_OK (negative slots skip their token and never collide).
 * Both return PKV_EINVAL for num < 0 or a null array with num > 0.
 *
 * pkv_set_debug_checks(enable): with enable = 1 (0), kv_block_copy and
 *   kv_cache_append run these checks on every call (do not); enable < 0 only
 *   queries.  Returns the setting before the call.  The initial setting is on
 *   when the environment variable PKV_CHECK is "1" at the first query, else off.
 *   A checked call synchronises its stream (the indices are device memory), so
 *   the checks are for debugging, not for a serving loop's hot path.
 */
int pkv_check_copy_pairs(const int64_t* host_pairs, int num_pairs);
int pkv_check_slots(const int64_t* host_slots, int num_tokens);
int pkv_set_debug_checks(int enable);

/*
 * paged_kv_gather - copy one sequence's cached rows into contiguous memory.
 *
 * out[h][t][:] = cache[block_table_row[t / B]][h][t % B][:] for t < context_len,
 * bit for bit, through the same address computation the decode kernel uses.
 * For checking block-table indexing and for exporting a sequence.
 *
 *   cache            one pool, [num_blocks][num_heads][block_size][head_dim].
 *   block_table_row  int32 [>= ceil(context_len / block_size)], device memory.
 *   context_len      host int, >= 0.
 *   out              [num_heads][context_len][head_dim], storage dtype.
 */
int paged_kv_gather(const void* cache, const int32_t* block_table_row, int context_len,
                    int num_heads, int head_dim, int block_size, int num_blocks,
                    pkv_dtype dtype, void* out, void* stream);

/*
 * kv_blocks_to_host / kv_blocks_from_host - block-granular swap of the cache to and
 * from pinned host memory (a preempted sequence's blocks move to host RAM and back:
 * "PagedAttention - Efficient Memory Management for LLM Serving with vLLM", section
 * "Method", scheduling).
 *
 *   to host:   host_k[i] = k_cache[block_ids[i]] and host_v[i] = v_cache[block_ids[i]]
 *   from host: k_cache[block_ids[i]] = host_k[i] and v_cache[block_ids[i]] = host_v[i]
 * for i < num_blocks_moved, every head and slot, bit for bit, in one kernel launch
 * that reads or writes host memory directly over the host link.
 *
 *   block_ids     int64 [num_blocks_moved], device memory.
 *   host_k,
 *   host_v        pinned (page-locked) host memory, [num_blocks_moved][num_heads]
 *                 [block_size][head_dim] each, 16-byte aligned; memory that is not
 *                 page-locked is rejected with PKV_EINVAL.
 * An id outside [0, num_blocks) is skipped and flagged (PKV_DEV_COPY_PAIR).  The
 * host buffers must not be touched by the host until the stream has passed the call.
 */
int kv_blocks_to_host(const void* k_cache, const void* v_cache, const int64_t* block_ids,
                      int num_blocks_moved, void* host_k, void* host_v, int num_heads,
                      int head_dim, int block_size, int num_blocks, pkv_dtype dtype, void* stream);
int kv_blocks_from_host(const void* host_k, const void* host_v, void* k_cache, void* v_cache,
                        const int64_t* block_ids, int num_blocks_moved, int num_heads,
                        int head_dim, int block_size, int num_blocks, pkv_dtype dtype,
                        void* stream);

/*
 * Block manager: host bookkeeping of the physical block pool (pure host code, no
 * CUDA call).  Blocks come from the front of a FIFO free list with reference count
 * 1 and return to its back when the count reaches 0 ("vLLM PagedAttention and
 * continuous batching", section 4); a sequence of n tokens holds ceil(n / B)
 * blocks, taken on demand ("LLM Inference 8 - PagedAttention", section
 * "PagedAttention의 동작 방식"); forked sequences share blocks, and an append into a
 * shared last block copies it first (copy-on-write, the paper digest's flowchart).
 * Calls on one manager are serialised by an internal mutex.  Sequence ids are any
 * int64 values.  Errors: PKV_EINVAL (bad argument), PKV_ESEQ, PKV_ENOMEM; a failed
 * call changes nothing.
 */
typedef struct pkv_block_manager pkv_block_manager;

/* free_order: NULL for 0, 1, ..., num_blocks - 1, else a permutation of them. NULL on bad arguments. */
pkv_block_manager* pkv_bm_create(int num_blocks, int block_size, const int32_t* free_order);
void pkv_bm_destroy(pkv_block_manager* bm);
/* A new sequence holding num_tokens tokens (a prompt): takes ceil(num_tokens / B) blocks. */
int pkv_bm_add_sequence(pkv_block_manager* bm, int64_t seq, int num_tokens);
/* child shares every block of parent (reference counts + 1). */
int pkv_bm_fork(pkv_block_manager* bm, int64_t parent, int64_t child);
/*
 * One new token for each of the n distinct sequences: slots[i] receives the slot of
 * seqs[i]'s new token (for kv_cache_append); each copy-on-write appends its
 * (src, dst) pair to cow_pairs (capacity 2 * n entries; for kv_block_copy) and
 * *num_pairs counts them.
 */
int pkv_bm_append_tokens(pkv_block_manager* bm, const int64_t* seqs, int n, int64_t* slots,
                         int64_t* cow_pairs, int* num_pairs);
/* Releases the sequence's blocks (or forgets a swapped-out sequence). */
int pkv_bm_free_sequence(pkv_block_manager* bm, int64_t seq);
/* Copies the block table (padded with -1 to max_blocks) and the token count; returns the block count. */
int pkv_bm_block_table(pkv_block_manager* bm, int64_t seq, int32_t* row, int max_blocks,
                       int64_t* num_tokens);
/* Block tables [n][max_blocks] and context lengths [n] of n sequences: the decode step's inputs. */
int pkv_bm_fill_tables(pkv_block_manager* bm, const int64_t* seqs, int n, int32_t* block_tables,
                       int max_blocks, int32_t* context_lens);
int pkv_bm_num_free(pkv_block_manager* bm);
int pkv_bm_ref_count(pkv_block_manager* bm, int block);
/* Lists the sequence's blocks in logical order (copy them with kv_blocks_to_host), then releases them. */
int pkv_bm_swap_out(pkv_block_manager* bm, int64_t seq, int64_t* blocks, int max_blocks, int* n_blocks);
/* Takes fresh blocks for a swapped-out sequence: host slot i goes to blocks[i] (kv_blocks_from_host). */
int pkv_bm_swap_in(pkv_block_manager* bm, int64_t seq, int64_t* blocks, int max_blocks, int* n_blocks);

/*
 * pkv_selftest_wait_timeout - exercise the bounded-wait path that every pipeline
 * wait in the attention kernels uses (no counterpart on the pages: failure
 * detection for the library itself).  Launches one CTA on `stream` whose thread 0
 * waits on a fresh shared-memory mbarrier that nothing arrives on, bounded by
 * `limit_cycles` SM clock cycles (1 ... 2e9, the kernels' own bound); the wait runs
 * out, the kernel records PKV_DEV_WAIT_TIMEOUT in the device error word and returns
 * normally, so the context stays usable.  Synchronises the stream.  Returns 1 when
 * the wait ran out, 0 if it completed (it cannot), PKV_EINVAL for a limit out of
 * range (checked on the host, nothing launched) or PKV_ECUDA.  Read and clear the
 * recorded reason with pkv_get_device_error.
 */
int pkv_selftest_wait_timeout(long long limit_cycles, void* stream);

/*
 * pkv_get_device_error - synchronise `stream`, read and clear the device error
 * word of the current device.  Returns PKV_OK when it was clear, PKV_ETIMEOUT when
 * it records PKV_DEV_WAIT_TIMEOUT, PKV_EDEVICE for any other reason, PKV_ECUDA if
 * the synchronisation or the read failed.  *reason (may be NULL) receives the
 * first PKV_DEV_* reason recorded since the last clear.
 */
int pkv_get_device_error(void* stream, int* reason);

/* Static description of a return code. */
const char* pkv_strerror(int code);

/* ABI version of this header (incremented on incompatible changes). */
int pkv_abi_version(void);

/*
 * paged_attn_decode_noalloc - paged_attn_decode for callers that cannot allocate.
 *
 * The pages have no counterpart to this entry point; it exists for integration.
 * Some callers are handed only a stream and their own input/output buffers by a
 * host framework that owns every byte of device memory (plugin-style backends),
 * and some run latency-critical loops where a cudaMalloc, with its implicit
 * device synchronisation and its chance of failing mid-step, is not acceptable.
 * Neither can provide the workspace paged_attn_decode needs.  This variant
 * computes exactly what paged_attn_decode computes, with the same arguments minus
 * the workspace, and takes its scratch (work list, partial softmax states) from a
 * static device array inside the library instead.  It calls no cudaMalloc,
 * cudaFree, cudaMallocAsync or other allocating routine.
 *
 *  - Size limit: the scratch array holds PKV_NOALLOC_SCRATCH_BYTES (32 MiB).  A
 *    call whose paged_attn_decode_workspace_size() exceeds it is rejected with
 *    PKV_EWORKSPACE before anything is launched.  Every GPU that loads the
 *    library holds this array until the process exits.
 *  - Set-up: the first call on a device, with that device current, looks up the
 *    array's device address (cudaGetSymbolAddress) and caches it; make that
 *    first call on each device before any stream capture begins.
 *  - Sharing: every call on a device uses the same array.  The call resets what
 *    must start at zero (the work counter) itself, and the array keeps the last
 *    call's contents.  Calls whose kernels overlap on the GPU (other streams,
 *    other host threads) race on the array: order them on one stream.
 *  - Return codes and device-side checks are those of paged_attn_decode given a
 *    workspace of PKV_NOALLOC_SCRATCH_BYTES: the same argument checks run in the
 *    same order (dtype, sizes, scale, then pointers and alignment; num_seqs = 0
 *    returns PKV_OK after the size checks), and PKV_EWORKSPACE comes last.
 */
#define PKV_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)
int paged_attn_decode_noalloc(const void* q, const void* k_cache, const void* v_cache,
                              const int32_t* block_tables, const int32_t* context_lens,
                              int num_seqs, int num_heads, int head_dim, int block_size,
                              int max_blocks_per_seq, int num_blocks, pkv_dtype dtype,
                              float scale, float* out, int partition_tokens, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* PAGEDKV_H_ */
