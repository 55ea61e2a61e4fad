/*
 * pagedattn.h -- C ABI of the paged KV-cache decode path (sm_100a).
 *
 * The method ("PagedAttention Internals", wondering.app, sections "Fixed-Size
 * KV Blocks" and "The Block Table Map"; "pagedattention" glossary entry,
 * chipfoundryservices.com, paragraph 3 on block tables): every sequence's
 * key/value cache is stored in fixed-size physical blocks that may sit
 * anywhere in a shared pool, and a per-sequence block table maps logical block
 * n to its physical block.  The attention step reads through the table; new
 * tokens fill the sequence's current block and a new block is taken only when
 * it is full; sequences that share a prefix (or the samples of a beam search)
 * point at the same physical blocks, which are copied only when a sharer
 * writes into them (glossary entry, comparison table and paragraph 5 on
 * sharing).
 *
 * Conventions for every entry point:
 *  - Pointers named "device" are CUDA device pointers owned by the caller;
 *    pointers named "host" are host memory owned by the caller.  The library
 *    never allocates, frees or keeps device memory of the caller's.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream).  Kernel launches are asynchronous on it; no call synchronises
 *    except pa_read_device_error.
 *  - Every call returns a pa_status.  Argument errors are found on the host
 *    before any launch and leave every buffer untouched.
 *  - Data errors that only the device can see (a slot or a table entry
 *    outside the pool) never trap: the offending element is skipped and a
 *    bit is set in a per-device error word read by pa_read_device_error.
 *  - A kernel of this library may start while the library kernel ahead of
 *    it on the same stream is still running (programmatic dependent
 *    launch); it waits for that kernel before it reads or writes anything
 *    the kernel may touch.  The one exception: the tensor-core pa_decode
 *    reads context_lens and block_tables before that wait.  No kernel of the
 *    library writes int32 tables or lengths, so this only forbids placing
 *    them in memory that the preceding library call writes (a pool, an
 *    output or a workspace).
 *
 * Cache layout (both pools):
 *   k_cache, v_cache : [num_blocks][num_kv_heads][block_size][head_dim]
 *   element (blk, h, off, d) at ((blk*num_kv_heads + h)*block_size + off)*head_dim + d,
 *   so one (block, kv head) tile of block_size x head_dim is contiguous.
 * A token at logical position t of a sequence with block table T lives at
 *   slot = T[t / block_size] * block_size + t % block_size.
 */
#ifndef PAGEDATTN_H
#define PAGEDATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define PA_API __attribute__((visibility("default")))
#else
#define PA_API
#endif

typedef enum {
  PA_OK = 0,
  PA_ERR_INVALID_ARG = 1,   /* a null pointer, a bad size or shape */
  PA_ERR_UNSUPPORTED = 2,   /* dtype / head_dim / block_size / group size not built */
  PA_ERR_OUT_OF_BLOCKS = 3, /* allocator: not enough free blocks; state unchanged */
  PA_ERR_CUDA = 4,          /* a CUDA runtime call failed */
  PA_ERR_NOT_FOUND = 5,     /* allocator: no such live sequence */
  PA_ERR_TOO_SMALL = 6      /* a caller buffer (workspace, table row, output) is too small */
} pa_status;

typedef enum { PA_DTYPE_F32 = 0, PA_DTYPE_BF16 = 1 } pa_dtype;

/* Bits of the device error word (pa_read_device_error). */
#define PA_DEVERR_SLOT 0x1       /* pa_append_kv: slot >= num_blocks*block_size (row skipped) */
#define PA_DEVERR_TABLE 0x2      /* pa_decode: a used table entry outside [0, num_blocks) (block skipped) */
#define PA_DEVERR_PAIR 0x4       /* pa_copy_blocks: a pair entry outside [0, num_blocks) (pair skipped) */
#define PA_DEVERR_TIMEOUT 0x8    /* a kernel gave up waiting on its own copy (work unit dropped) */
#define PA_DEVERR_LEN 0x10       /* pa_decode: a context length < 0 or > max_context_len (row zeroed) */
#define PA_DEVERR_PLAN 0x20      /* pa_decode_shared: a sharing plan entry that does not fit its sequence (ignored) */

/* Tokens per split-context partition of the decode calls unless the pool
 * says otherwise (pa_cache_t.partition_tokens). */
#define PA_PARTITION_TOKENS 512

/* The paged pool.  k and v are device pointers of the layout above. */
typedef struct {
  void *k;
  void *v;
  int32_t dtype;        /* pa_dtype of every element of k, v, q, out and the new rows */
  int32_t num_blocks;
  int32_t block_size;   /* tokens per block: 8, 16 or 32 */
  int32_t num_kv_heads;
  int32_t head_dim;     /* 64 or 128 */
  /* Tokens per split-context partition of the decode calls over this pool:
   * 256, 512 or 1024, or 0 for PA_PARTITION_TOKENS.  It sets the workspace
   * size (pa_decode_workspace_size_p, pa_decode_shared_workspace_size). */
  int32_t partition_tokens;
} pa_cache_t;

/* ---------------------------------------------------------------- kernels */

/*
 * KV append ("Fixed-Size KV Blocks": tokens fill the current block; the
 * glossary's paragraph 3: the table maps logical positions to physical
 * blocks).
 *   k, v          device [num_tokens][num_kv_heads][head_dim], cache dtype
 *   slot_mapping  device [num_tokens] int64: token i is written to
 *                 k_cache/v_cache[slot/bs][h][slot%bs][:] for every head h.
 *                 A negative slot is padding and is skipped; a slot past the
 *                 pool sets PA_DEVERR_SLOT and is skipped.
 * Two tokens with the same slot: which one lands is undefined.
 */
PA_API pa_status pa_append_kv(const void *k, const void *v, const int64_t *slot_mapping,
                              int32_t num_tokens, const pa_cache_t *cache, void *stream);

/*
 * Paged decode attention ("The Block Table Map" and the glossary's paragraph
 * 3: the attention step gathers each sequence's keys and values through its
 * block table).  The pages give no formula; this is the textbook scaled
 * dot-product step.  For sequence b, query head h and its KV head
 * g = h / (num_q_heads / num_kv_heads):
 *   s_t = scale * <q[b,h,:], K(b,t,g)>  for t < context_lens[b]
 *   out[b,h,:] = sum_t exp(s_t - max s) V(b,t,g) / sum_t exp(s_t - max s)
 * with K(b,t,g) = k_cache[block_tables[b*max_blocks_per_seq + t/bs]][g][t%bs].
 * Contexts are cut into partitions of the pool's partition_tokens; each partition
 * keeps (max, sum, unnormalised accumulator) in the workspace and a second
 * kernel merges them with a log-sum-exp combine.  Arithmetic is fp32 with an
 * online softmax; out is rounded once to the cache dtype.
 *   q             device [num_seqs][num_q_heads][head_dim], cache dtype
 *   block_tables  device [num_seqs][max_blocks_per_seq] int32; entries past
 *                 ceil(len/bs) are never read
 *   context_lens  device [num_seqs] int32 (the appended token included);
 *                 0 gives a zero output row
 *   max_context_len  host: an upper bound of every context_lens[b]; a larger
 *                 length sets PA_DEVERR_LEN and zeroes that row
 *   out           device [num_seqs][num_q_heads][head_dim], cache dtype
 *   workspace     device scratch of at least pa_decode_workspace_size_p(...,
 *                 cache->partition_tokens) bytes, 16-byte aligned (NULL
 *                 allowed when that size is 0)
 * num_q_heads / num_kv_heads (the group size) must be 1, 2, 4 or 8.
 */
PA_API pa_status pa_decode(const void *q, const pa_cache_t *cache, const int32_t *block_tables,
                           int32_t max_blocks_per_seq, const int32_t *context_lens,
                           int32_t num_seqs, int32_t num_q_heads, int32_t max_context_len,
                           float scale, void *out, void *workspace, size_t workspace_bytes,
                           void *stream);

/*
 * One decode step in one call: for every sequence b, the copy-on-write copy
 * of its last block (when cow_src asks for one), the append of its newest
 * token, and pa_decode over the updated pool.  The pages describe the three
 * as the steps a sequence takes when it grows ("Fixed-Size KV Blocks": a
 * token goes into the current block; glossary paragraph 5: a shared block is
 * copied when a sharer writes into it).  The result (pool and out) is
 * bit-for-bit that of
 *   pa_copy_blocks({cow_src[b], T_b[(len_b-1)/bs]} for every b with cow_src[b] >= 0)
 *   pa_append_kv(k_new, v_new, {T_b[(len_b-1)/bs]*bs + (len_b-1)%bs})
 *   pa_decode(q, ..., out)
 * with T_b the block table of b and len_b = context_lens[b]; on the
 * tensor-core path it is one launch (plus the log-sum-exp reduce), the
 * append and copy done by the CTA that reads the block afterwards.
 *   k_new, v_new  device [num_seqs][num_kv_heads][head_dim], cache dtype:
 *                 the key/value rows of token len_b - 1 of sequence b
 *   cow_src       device [num_seqs] int32, or NULL for no copies: a block
 *                 whose tiles (every kv head) are first copied over b's last
 *                 block, -1 for none.  A source outside the pool sets
 *                 PA_DEVERR_PAIR and is skipped.
 *   the rest      as pa_decode.
 * A sequence with len_b = 0 (or an invalid length) appends nothing.  Two
 * sequences must not have the same last block (a block that several
 * sequences share is copied for all writers but one), and a copy's source
 * must not be another sequence's copy destination.
 */
PA_API pa_status pa_append_decode(const void *k_new, const void *v_new, const int32_t *cow_src,
                                  const void *q, const pa_cache_t *cache,
                                  const int32_t *block_tables, int32_t max_blocks_per_seq,
                                  const int32_t *context_lens, int32_t num_seqs,
                                  int32_t num_q_heads, int32_t max_context_len, float scale,
                                  void *out, void *workspace, size_t workspace_bytes,
                                  void *stream);

/*
 * A sharing plan for pa_decode_shared: groups of sequences of one batch whose
 * block tables hold the same physical blocks for their first
 * shared_tokens[j] tokens (whole blocks, every one of them before each
 * member's last block).  pa_share_plan builds one from host tables.
 *   members       device [n_groups][max_members] int32: sequence indices of
 *                 the batch, a group's members first, -1 after its last
 *   shared_tokens device [n_groups] int32 (> 0, a multiple of the block size)
 *   first_token   device [num_seqs] int32: shared_tokens[j] for a member of
 *                 group j, 0 for a sequence in no group
 *   max_members   1..4 (the cascade kernel's query tile holds 4 sequences)
 * A sequence belongs to at most one group.  If the tables of a group do not
 * agree on those blocks the results are undefined; a first_token that is
 * not a multiple of the block size or not below its sequence's length sets
 * PA_DEVERR_PLAN and that sequence is computed whole.
 */
/* Shared prefixes shorter than this are not worth a cascade unit. */
#define PA_SHARE_MIN_TOKENS 128

typedef struct {
  const int32_t *members;
  const int32_t *shared_tokens;
  const int32_t *first_token;
  int32_t n_groups;
  int32_t max_members;
} pa_share_plan_t;

/*
 * pa_decode (or pa_append_decode, when k_new and v_new are given) with a
 * cascade over shared blocks: the prefix a plan's group shares is read once
 * for all its members ("pagedattention" glossary entry, paragraph 5:
 * sequences that share a prefix point at the same physical blocks;
 * "PagedAttention Internals", "Sharing And Dynamic Growth").  The cascade
 * computes each member's statistics over the shared prefix in pieces of the
 * pool's partitions; when a prefix ends inside a partition, that partition's
 * statistics come in two parts (the shared piece, kept in an extra workspace
 * row, and the member's own rest), which the log-sum-exp reduce merges with
 * the others.  The result is the same attention: within the decode's
 * tolerances of pa_decode / pa_append_decode, and bit for bit when every
 * group's prefix ends on a partition boundary.  plan may be NULL or have no
 * groups; on the CUDA-core path (not bf16 with head_dim 128) the plan is not
 * used and every sequence computes all of its partitions.
 *   k_new, v_new, cow_src  as pa_append_decode, or all NULL for no append
 *   plan                   host pointer to the plan (its arrays on the device)
 *   workspace              with a plan that has groups: at least
 *                          pa_decode_shared_workspace_size(...) bytes
 *   the rest               as pa_decode
 */
PA_API pa_status pa_decode_shared(const void *k_new, const void *v_new, const int32_t *cow_src,
                                  const void *q, const pa_cache_t *cache,
                                  const int32_t *block_tables, int32_t max_blocks_per_seq,
                                  const int32_t *context_lens, int32_t num_seqs,
                                  int32_t num_q_heads, int32_t max_context_len, float scale,
                                  const pa_share_plan_t *plan, void *out, void *workspace,
                                  size_t workspace_bytes, void *stream);

/*
 * Paged chunked-prefill attention: the decode step of "The Block Table Map"
 * for every new token of a chunk, with a causal limit.  Sequence b holds
 * context_lens[b] tokens in the cache (the chunk's own rows appended with
 * pa_append_kv first); the last n_b = query_starts[b+1] - query_starts[b] of
 * them are new, and new token i (position context_lens[b] - n_b + i) attends
 * to the sequence's tokens 0 .. its own position:
 *   out[query_starts[b] + i][h] = softmax_t(scale <q[...][h], K(b,t,g)>) . V(b,t,g), t <= position
 * with g = h / (num_q_heads / num_kv_heads).  bf16, head_dim 128 only
 * (PA_ERR_UNSUPPORTED otherwise); fp32 accumulation, out rounded once.
 *   q             device [total_query_tokens][num_q_heads][128] bf16
 *   query_starts  device [num_seqs + 1] int32, query_starts[0] = 0, ascending,
 *                 query_starts[num_seqs] = total_query_tokens
 *   block_tables, context_lens, max_context_len  as pa_decode
 *   max_query_len host: an upper bound of every n_b (sizes the grid)
 *   out           device [total_query_tokens][num_q_heads][128] bf16
 * A sequence with n_b > context_lens[b] or a length past max_context_len
 * sets PA_DEVERR_LEN and writes nothing; a used table entry outside the pool
 * sets PA_DEVERR_TABLE (that sequence's rows are then undefined).
 */
PA_API pa_status pa_prefill(const void *q, const pa_cache_t *cache, const int32_t *block_tables,
                            int32_t max_blocks_per_seq, const int32_t *context_lens,
                            const int32_t *query_starts, int32_t num_seqs, int32_t num_q_heads,
                            int32_t total_query_tokens, int32_t max_query_len,
                            int32_t max_context_len, float scale, void *out, void *stream);

/* Bytes of workspace pa_decode needs for these sizes with partitions of
 * PA_PARTITION_TOKENS tokens (0 when no context is longer than one
 * partition). */
PA_API size_t pa_decode_workspace_size(int32_t num_seqs, int32_t num_q_heads,
                                       int32_t max_context_len, int32_t head_dim);

/* The same for partitions of partition_tokens tokens (256, 512 or 1024; 0
 * for PA_PARTITION_TOKENS); 0 for any other size. */
PA_API size_t pa_decode_workspace_size_p(int32_t num_seqs, int32_t num_q_heads,
                                         int32_t max_context_len, int32_t head_dim,
                                         int32_t partition_tokens);

/* Bytes of workspace pa_decode_shared needs with a sharing plan that has
 * groups: one more row per (sequence, query head) than pa_decode (the
 * shared piece of the partition a prefix ends in), and some even when no
 * context is longer than one partition.  0 for an unsupported size. */
PA_API size_t pa_decode_shared_workspace_size(int32_t num_seqs, int32_t num_q_heads,
                                              int32_t max_context_len, int32_t head_dim,
                                              int32_t partition_tokens);

/*
 * pa_decode without a caller-provided workspace.  The pages have no
 * counterpart: this is a convenience of this library for callers that cannot
 * allocate device memory at decode time -- for example a serving process that
 * has handed nearly all of HBM to the paged KV pool (the pool is normally
 * sized to fill whatever memory is left, so a workspace allocation can fail),
 * or code running behind a plugin or runtime interface that offers no device
 * allocator.  It allocates nothing: the split-context scratch lives in one
 * fixed array of PA_STATIC_WORKSPACE_BYTES inside the library, which every
 * GPU that loads the library holds until the process exits.
 *  - Arguments and results are those of pa_decode (minus the workspace).
 *  - Sizes whose scratch, pa_decode_workspace_size_p(num_seqs, num_q_heads,
 *    max_context_len, head_dim, partition), exceeds PA_STATIC_WORKSPACE_BYTES are
 *    rejected with PA_ERR_TOO_SMALL before any launch (with the pool's
 *    partition_tokens: pa_decode_workspace_size_p).
 *  - The first call in a CUDA context looks up that context's copy of the
 *    array (with the context current, the runtime's current device's
 *    primary context unless the caller bound another); make that first call
 *    before any stream capture.  Later calls in the same context reuse the
 *    address.  The address is tied to the context it was looked up in: a
 *    context created later (another context of the device, or the primary
 *    context again after cudaDeviceReset) gets a lookup of its own.
 *  - Every call on a device shares the one array and it keeps the last call's
 *    contents.  Nothing in it needs to start at zero: each entry the merge
 *    step reads is written earlier in the same call.  Calls whose kernels
 *    overlap on the GPU (different streams, no ordering between them) race
 *    on the array and may return wrong results; order them on one stream.
 */
#define PA_STATIC_WORKSPACE_BYTES (8u << 20)

PA_API pa_status pa_decode_static_workspace(const void *q, const pa_cache_t *cache,
                                            const int32_t *block_tables,
                                            int32_t max_blocks_per_seq,
                                            const int32_t *context_lens, int32_t num_seqs,
                                            int32_t num_q_heads, int32_t max_context_len,
                                            float scale, void *out, void *stream);

/*
 * Copy-on-write block copy (glossary entry, comparison table row on sharing
 * and paragraph 5: sharers get their own copy of a block only when they
 * diverge).  For every pair i, physical block
 * src_dst_pairs[2i+1] of both pools becomes a bit copy of block
 * src_dst_pairs[2i] (all kv heads, all slots).
 *   src_dst_pairs device [num_pairs][2] int32
 * Destinations must be distinct and no destination may also be a source
 * (pa_check_copy_pairs tests this on a host copy); otherwise the result is
 * undefined.  An entry outside the pool sets PA_DEVERR_PAIR; that pair is
 * skipped.
 */
PA_API pa_status pa_copy_blocks(const int32_t *src_dst_pairs, int32_t num_pairs,
                                const pa_cache_t *cache, void *stream);

/* Host-side check of copy pairs (host memory): PA_OK, or PA_ERR_INVALID_ARG
 * for an entry outside [0, num_blocks), a repeated destination, or a
 * destination that is also a source. */
PA_API pa_status pa_check_copy_pairs(const int32_t *src_dst_pairs_host, int32_t num_pairs,
                                     int32_t num_blocks);

/* Synchronises `stream`, then returns the current device's error word in
 * *bits (PA_DEVERR_*) and clears it. */
PA_API pa_status pa_read_device_error(void *stream, int32_t *bits);

/* Synchronises `stream` and returns (and clears) where the first wait that
 * gave up since the last call was (the cause of PA_DEVERR_TIMEOUT):
 * info[0] = 1 if any, info[1] = the shared-memory address of its mbarrier,
 * info[2] = its phase parity | block index << 1, info[3] = thread index. */
PA_API pa_status pa_read_wait_timeout(void *stream, uint32_t info[4]);

/* Static text for a status code. */
PA_API const char *pa_status_string(pa_status s);

/* The cudaError_t of the CUDA call behind the calling thread's most recent
 * PA_ERR_CUDA from this library (0 if there was none), and CUDA's static
 * text for such a code. */
PA_API int32_t pa_last_cuda_error(void);
PA_API const char *pa_cuda_error_string(int32_t code);

/* Library version, "major.minor.patch". */
PA_API const char *pa_version(void);

/* ------------------------------------------------------ block allocator */
/*
 * Host-side reference-counted block allocator ("Fixed-Size KV Blocks",
 * "Sharing And Dynamic Growth"; glossary "Paging maps ..." and "It is the
 * core of vLLM ...").  Blocks are handed out one at a time as sequences
 * grow; forks share every block (reference count + 1); a write into a shared,
 * partially filled last block first moves the writer to a fresh block and
 * reports a (src, dst) copy pair for pa_copy_blocks; freed blocks return to
 * the pool.  The free list deals never-used blocks in a caller-given order
 * and hands released blocks out again last-in first-out.  Sequence ids are
 * never reused.  Not thread-safe: one allocator per host thread.
 */
typedef struct pa_allocator pa_allocator;

/* free_order_host: a permutation of [0, num_blocks) (the order fresh blocks
 * are dealt), or NULL for 0, 1, 2, ... */
PA_API pa_status pa_alloc_create(int32_t num_blocks, int32_t block_size,
                                 const int32_t *free_order_host, pa_allocator **out);
PA_API void pa_alloc_destroy(pa_allocator *a);

/* A new, empty sequence; its id in *seq. */
PA_API pa_status pa_seq_new(pa_allocator *a, int32_t *seq);

/* A new sequence sharing every block of `parent` (reference counts + 1). */
PA_API pa_status pa_seq_fork(pa_allocator *a, int32_t parent, int32_t *child);

/* Releases a sequence: reference counts - 1, blocks reaching 0 are freed. */
PA_API pa_status pa_seq_free(pa_allocator *a, int32_t seq);

/*
 * Appends n tokens to one sequence.  out_slots_host[n] receives each token's
 * slot.  A copy-on-write move, if any, is written to out_cow_pair_host[2]
 * (src, dst) and *n_cow is 1, else 0.  PA_ERR_OUT_OF_BLOCKS leaves every
 * state unchanged.
 */
PA_API pa_status pa_seq_append(pa_allocator *a, int32_t seq, int32_t n, int64_t *out_slots_host,
                               int32_t *out_cow_pair_host, int32_t *n_cow);

/*
 * Appends n_tokens[i] tokens to seqs[i] for every i, in order, all or nothing
 * (a sequence may appear once).  Slots go to out_slots_host, sequence by
 * sequence (sum of n_tokens entries); copy pairs to out_cow_pairs_host
 * (room for n_seqs pairs), *n_cow of them, in the order they were made.
 */
PA_API pa_status pa_batch_append(pa_allocator *a, const int32_t *seqs, const int32_t *n_tokens,
                                 int32_t n_seqs, int64_t *out_slots_host,
                                 int32_t *out_cow_pairs_host, int32_t *n_cow);

/* Length in tokens and number of blocks of a live sequence. */
PA_API pa_status pa_seq_len(pa_allocator *a, int32_t seq, int32_t *len, int32_t *num_blocks);

/* Copies a sequence's table into out_host (room for cap entries). */
PA_API pa_status pa_seq_block_table(pa_allocator *a, int32_t seq, int32_t *out_host, int32_t cap,
                                    int32_t *count);

/* The longest of n_seqs sequences: its length in tokens (the max_context_len
 * pa_decode takes) and its number of blocks (the narrowest table width). */
PA_API pa_status pa_seqs_max_len(pa_allocator *a, const int32_t *seqs, int32_t n_seqs,
                                 int32_t *max_len, int32_t *max_blocks);

/* Writes the tables of n_seqs sequences as rows of a [n_seqs][max_blocks]
 * int32 host array padded with `pad`, and their lengths to lens_host. */
PA_API pa_status pa_build_block_tables(pa_allocator *a, const int32_t *seqs, int32_t n_seqs,
                                       int32_t max_blocks, int32_t pad, int32_t *tables_host,
                                       int32_t *lens_host);

/* Usage: slots holding a token (each physical slot once), slots allocated
 * (blocks in use x block_size), free and used block counts.  Fragmentation
 * = (allocated - used) / allocated. */
PA_API pa_status pa_alloc_stats(pa_allocator *a, int64_t *used_slots, int64_t *allocated_slots,
                                int32_t *free_blocks, int32_t *used_blocks);

/* Reference count of a physical block. */
PA_API pa_status pa_block_refcount(pa_allocator *a, int32_t block, int32_t *refcount);

/*
 * Builds a sharing plan from host tables (after the step's appends):
 * sequences with a block before their last one whose first table entries
 * are the same physical block form buckets (sharers point at the same blocks
 * from the start); each bucket is cut into groups of at most max_members
 * (2..4) in sequence order, a lone leftover joins no group; a group shares
 * the leading blocks on which all its members' tables agree, each before
 * every member's last block, and is kept when that is at least
 * PA_SHARE_MIN_TOKENS tokens.
 *   tables_host  [n_seqs][max_blocks] int32, lens_host [n_seqs] int32
 *   members_host room for n_seqs / 2 groups x max_members, -1 padded
 *   shared_host  room for n_seqs / 2: each group's shared tokens
 *   first_token_host [n_seqs]
 */
PA_API pa_status pa_share_plan(const int32_t *tables_host, int32_t max_blocks,
                               const int32_t *lens_host, int32_t n_seqs, int32_t block_size,
                               int32_t max_members, int32_t *members_host, int32_t *shared_host,
                               int32_t *first_token_host, int32_t *n_groups);

/*
 * One decode step's host work in one call: appends one token to each of the
 * n_seqs sequences (all or nothing, as pa_batch_append; PA_ERR_OUT_OF_BLOCKS
 * leaves every state unchanged), then writes what pa_decode_shared takes:
 *   tables_host [n_seqs][max_blocks] and lens_host [n_seqs] after the
 *     append; a row's entries past the sequence's blocks are not written (no
 *     kernel reads them); PA_ERR_TOO_SMALL before any change when a table
 *     would not fit max_blocks;
 *   cow_src_host [n_seqs]: the block a sequence's copy-on-write move copies
 *     into its new last block, -1 for none (*n_copies of them);
 *   with share_max_members in 2..4, the sharing plan of pa_share_plan
 *     (members_host room for n_seqs / 2 groups x share_max_members,
 *     shared_host room for n_seqs / 2, *n_groups); with 0, no plan and
 *     first_token_host all zeros;
 *   *max_len: the longest length (max_context_len of the call).
 */
PA_API pa_status pa_decode_step_prepare(pa_allocator *a, const int32_t *seqs, int32_t n_seqs,
                                        int32_t max_blocks, int32_t share_max_members,
                                        int32_t *tables_host, int32_t *lens_host,
                                        int32_t *cow_src_host, int32_t *members_host,
                                        int32_t *shared_host, int32_t *first_token_host,
                                        int32_t *n_groups, int32_t *n_copies, int32_t *max_len);

/* ------------------------------------------------- one decode step, end to end */
/*
 * A whole decode step from host memory in one call, for serving loops that
 * hold their queries and new key/value rows in pinned host buffers: the
 * step's host work (pa_decode_step_prepare: one token per sequence through
 * the allocator, the tables, lengths, copy-on-write sources and sharing
 * plan), one host-to-device copy of every input, pa_decode_shared (copy on
 * write, append, decode), and the device-to-host copy of the output.  The
 * pages describe these as what each step of a growing sequence does
 * ("Fixed-Size KV Blocks": the new token goes into the current block, a
 * block is taken only when it is full; "pagedattention" glossary entry,
 * paragraph 5: shared blocks are copied when a sharer writes).
 *
 * A step slot holds one step's buffers; alternating two slots lets the host
 * prepare step i + 1 while the device runs step i.  Every buffer is the
 * caller's:
 *   host      pinned host staging area of pa_step_layout(...).bytes bytes:
 *             the caller writes q, k_new and v_new at their offsets before
 *             the call; the call writes the rest
 *   dev       device buffer of the same size (the staging area's mirror)
 *   out_host  pinned host [n_seqs][num_q_heads][head_dim], cache dtype
 *   out_dev   device, same shape
 *   workspace device scratch of pa_decode_shared_workspace_size(n_seqs,
 *             num_q_heads, max_blocks * block_size, head_dim,
 *             cache->partition_tokens) bytes (or more) with a plan
 *             (share_max_members > 0), else pa_decode_workspace_size_p(...)
 *   ev_in, ev_kernel, ev_out   CUDA events (cudaEvent_t) of the slot, made by
 *             pa_step_slot_events and released by pa_step_slot_release
 */
typedef struct {
  size_t q, k_new, v_new, tables, lens, cow_src, first_token, members, shared_tokens;  /* byte offsets */
  size_t bytes;                                                              /* total */
} pa_step_layout_t;

typedef struct {
  void *host;
  void *dev;
  void *out_host;
  void *out_dev;
  void *workspace;
  size_t workspace_bytes;
  void *ev_in;      /* recorded on h2d_stream once the inputs are on the device */
  void *ev_kernel;  /* recorded on stream once the decode has run */
  void *ev_out;     /* recorded on d2h_stream once out is on the host */
} pa_step_slot_t;

/* Offsets (16-byte aligned) of a step's inputs in the staging area:
 * q [n][Hq][D], k_new and v_new [n][Hkv][D] (cache dtype), tables
 * [n][max_blocks], lens [n], cow_src [n], first_token [n], members
 * [n / 2][share_max_members], shared_tokens [n / 2] (int32). */
PA_API pa_status pa_step_layout(int32_t n_seqs, int32_t num_q_heads, const pa_cache_t *cache,
                                int32_t max_blocks, int32_t share_max_members, pa_step_layout_t *layout);

/* Creates the slot's three events (timing disabled) on the current device. */
PA_API pa_status pa_step_slot_events(pa_step_slot_t *slot);
/* Destroys the slot's events (after the slot's last step is done). */
PA_API pa_status pa_step_slot_release(pa_step_slot_t *slot);
/* Blocks the host until the slot's last step has copied its inputs to the
 * device (its staging area may be rewritten) and its output to the host
 * (out_host holds that step's result).  A slot never used returns at once. */
PA_API pa_status pa_step_slot_wait(const pa_step_slot_t *slot);

/*
 * One decode step of n_seqs sequences (host ids seqs_host) through `slot`:
 *  1. pa_decode_step_prepare into the staging area (all or nothing: an
 *     error here, e.g. PA_ERR_OUT_OF_BLOCKS, leaves the allocator and the
 *     device untouched);
 *  2. on h2d_stream, after the slot's previous decode: one cudaMemcpyAsync
 *     of the staging area to dev, then ev_in;
 *  3. on stream, after ev_in and the slot's previous output copy:
 *     pa_decode_shared with the plan (share_max_members 2..4, or 0 for none),
 *     the copy sources and the new rows, then ev_kernel;
 *  4. on d2h_stream, after ev_kernel: cudaMemcpyAsync of out_dev to
 *     out_host, then ev_out.
 * Nothing is synchronised: call pa_step_slot_wait(slot) before rewriting
 * the slot's staging area or reading its out_host.  Any of the three
 * streams may be the same stream; with three distinct streams the copies of
 * step i + 1 in and of step i out run beside the decodes (a copy stream
 * shared by both directions would put step i + 1's inputs behind step i's
 * output, and so behind step i's decode).  *n_copies, *n_groups and *max_len report the
 * step's copies on write, plan groups and longest context.  A CUDA error
 * after step 1 returns PA_ERR_CUDA with the allocator already advanced.
 */
PA_API pa_status pa_decode_step(pa_allocator *a, const int32_t *seqs_host, int32_t n_seqs,
                                int32_t max_blocks, int32_t share_max_members,
                                const pa_cache_t *cache, int32_t num_q_heads, float scale,
                                const pa_step_slot_t *slot, void *stream, void *h2d_stream,
                                void *d2h_stream,
                                int32_t *n_copies, int32_t *n_groups, int32_t *max_len);

/*
 * The per-sequence form of a decode step's copy pairs, as pa_append_decode
 * takes it.  Sequence i's last block is the table entry of its newest token,
 * tables_host[i][(lens_host[i] - 1) / block_size] ("The Block Table Map":
 * logical block n of a sequence is entry n of its table); cow_src_host[i] is
 * the source of the pair whose destination is that block, else -1 (also
 * for lens_host[i] <= 0, a sequence with no block).
 *   pairs_host   [n_pairs][2] int32 (src, dst), as the allocator made them
 *   tables_host  [n_seqs][max_blocks] int32, lens_host [n_seqs] int32: the
 *                step's tables and lengths after its appends
 * PA_ERR_INVALID_ARG when a destination repeats, when a pair's destination
 * is no sequence's last block (a pair the one-token step cannot make), or
 * when a newest token's entry lies past max_blocks.
 */
PA_API pa_status pa_cow_sources(const int32_t *pairs_host, int32_t n_pairs,
                                const int32_t *tables_host, int32_t max_blocks,
                                const int32_t *lens_host, int32_t n_seqs, int32_t block_size,
                                int32_t *cow_src_host);

/*
 * Internal fragmentation of the pool as it stands: the share of allocated
 * slots (blocks in use x block_size) that hold no token, (allocated - used) /
 * allocated with the counts of pa_alloc_stats (each physical slot once), 0
 * when no block is in use.  This is the measure of the learn-ml-visualized
 * chapter "inference-acceleration-pagedattention-vllm", fragmentation worked
 * example: waste = allocated - used, taken as a fraction of what is allocated.
 */
PA_API pa_status pa_alloc_fragmentation(pa_allocator *a, double *fragmentation);

#ifdef __cplusplus
}
#endif
#endif /* PAGEDATTN_H */
