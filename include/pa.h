/*
 * pa.h -- C ABI of libpa.so: paged KV cache and paged decode attention for
 * NVIDIA B200 (sm_100a).
 *
 * The method: the KV cache of each request is cut into fixed-size physical
 * blocks that need not be adjacent, and a per-request block table maps the
 * request's logical block index to a physical block ("Paged attention in
 * LLMs", sections "The fix: stop demanding one continuous run" and "Keeping
 * track: the block table").  Decode attention reads a request's keys and
 * values through that table, with the gather inside the kernel's tiling loop
 * (quiz page "PagedAttention (vLLM)", code sketch "Conceptual: PagedAttention
 * block lookup").
 *
 * Conventions for every call
 * --------------------------
 *  - Return value: PA_OK (0) or a negative pa_status.  No C++ exception
 *    crosses this boundary.  pa_last_error_string() describes the last
 *    failure of the calling thread.
 *  - bf16 data is passed as pa_bf16 (raw 16-bit storage of bfloat16).
 *  - Device pointers are owned by the caller; the library never allocates,
 *    frees or retains device memory.  They must be 16-byte aligned and the
 *    tensors contiguous in the stated layout.
 *  - Kernel calls are asynchronous on `stream` (a cudaStream_t / CUstream
 *    handle, NULL = legacy default stream).  Argument errors are reported
 *    before anything is launched.  A launch failure returns PA_ERR_CUDA.
 *    The kernels are launched with programmatic stream serialisation: a
 *    kernel may start while the one before it on the stream finishes, and
 *    waits for that kernel's completion before it touches any memory the
 *    call's arguments name, so stream order holds as usual.
 *  - Device-side checks (block ids outside the pool, a slot outside the
 *    pool, a length beyond the block table, a pipeline wait that timed out)
 *    never trap: the kernel skips the offending access and records a code
 *    in a device error word, read with pa_device_error().
 *
 * KV pool layout (one pool per layer):
 *      kv_pool[num_blocks][2][num_kv_heads][block_size][head_dim]   bf16
 *  index 0 on the second axis holds keys, 1 holds values.  The quiz page's
 *  sketch prints a layer axis after the K/V axis; here each layer owns its
 *  own pool, so that axis is the caller's loop.
 */
#ifndef PA_H_
#define PA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t pa_bf16;

typedef enum pa_status {
  PA_OK = 0,
  PA_ERR_INVALID = -1,     /* bad argument (null, negative, misaligned, too small) */
  PA_ERR_UNSUPPORTED = -2, /* valid but not compiled (head_dim, block_size, group) */
  PA_ERR_OOM = -3,         /* allocator: not enough free blocks; state unchanged */
  PA_ERR_CUDA = -4,        /* a CUDA runtime/driver call failed */
  PA_ERR_NOT_FOUND = -5,   /* allocator: unknown sequence id */
  PA_ERR_EXISTS = -6       /* allocator: sequence id already present */
} pa_status;

/* Device error word bits (pa_device_error). */
#define PA_DEVERR_BLOCK_ID 0x1     /* block table entry outside [0, num_blocks) */
#define PA_DEVERR_SLOT 0x2         /* slot_mapping entry beyond the pool */
#define PA_DEVERR_SEQ_LEN 0x4      /* seq_len beyond max_blocks_per_seq*block_size */
#define PA_DEVERR_WAIT_TIMEOUT 0x8 /* a pipeline wait ran out of its time limit */
#define PA_DEVERR_COPY_PAIR 0x10   /* copy_blocks pair outside the pool */

/* Library version, major*10000 + minor*100 + patch. */
int pa_version(void);

/* Message for the last non-OK status returned on this thread (static storage). */
const char* pa_last_error_string(void);

/* Read (and when clear != 0, reset) the device error word of the current
 * device.  Synchronous: waits for all prior work on the device.  *code_out
 * is an OR of PA_DEVERR_* bits, 0 when no check fired. */
int pa_device_error(int32_t* code_out, int clear);

/* --------------------------------------------------------------------------
 * pa_reshape_and_cache -- write new tokens' keys and values into their slots.
 *
 * "Paged attention in LLMs", section "The cache being stored": the cache
 * grows by one token's keys and values per step.  Slot s addresses
 * physical block s / block_size, row s % block_size (the quiz page's sketch).
 *
 *   for t in [0, num_tokens) with s = slot_mapping[t] >= 0, for every head h:
 *     kv_pool[s / bs][0][h][s % bs][:] = key[t][h][:]
 *     kv_pool[s / bs][1][h][s % bs][:] = value[t][h][:]
 *
 * key, value   : device bf16 [num_tokens][num_kv_heads][head_dim], contiguous.
 * kv_pool      : device bf16 pool (layout above), written in place.
 * slot_mapping : device int64 [num_tokens]; negative = padding, no write.
 *                A slot >= num_blocks*block_size is skipped and flags
 *                PA_DEVERR_SLOT.  Two tokens with one slot: unspecified
 *                which one lands (the writes race).
 * head_dim     : multiple of 8.  num_tokens == 0 is a no-op.
 * Bit-exact copy: no arithmetic is done on the data.
 * ------------------------------------------------------------------------ */
int pa_reshape_and_cache(const pa_bf16* key, const pa_bf16* value, pa_bf16* kv_pool,
                         const int64_t* slot_mapping, int num_tokens, int num_blocks,
                         int num_kv_heads, int block_size, int head_dim, void* stream);

/* --------------------------------------------------------------------------
 * pa_copy_blocks -- duplicate whole physical blocks (copy-on-write).
 *
 * Quiz page "PagedAttention (vLLM)", comparison table row "Beam search /
 * best of N: copy on write blocks", and "Paged attention in LLMs", section
 * "Sharing blocks": a block shared by several requests is copied before one
 * of them writes into it.
 *
 *   for i in [0, num_pairs): kv_pool[pairs[2i+1]] = kv_pool[pairs[2i]]
 *   (all of [2][num_kv_heads][block_size][head_dim])
 *
 * block_pairs : device int32 [num_pairs][2] as (src, dst).  Pairs run
 *               concurrently; the result equals in-order application when
 *               no dst is also another pair's src or dst (always true for
 *               pairs produced by pa_alloc_append*).  A pair outside
 *               [0, num_blocks) is skipped and flags PA_DEVERR_COPY_PAIR.
 * Bit-exact copy.  num_pairs == 0 is a no-op.
 * ------------------------------------------------------------------------ */
int pa_copy_blocks(pa_bf16* kv_pool, const int32_t* block_pairs, int num_pairs,
                   int num_blocks, int num_kv_heads, int block_size, int head_dim,
                   void* stream);

/* --------------------------------------------------------------------------
 * pa_decode -- single-token decode attention over the paged cache.
 *
 * Quiz page "PagedAttention (vLLM)", code sketch "Conceptual: PagedAttention
 * block lookup": for each logical position pos in [0, seq_len) the keys and
 * values come from physical block block_table[pos / block_size], row
 * pos % block_size, followed by standard scaled-dot-product attention; real
 * kernels fold the gather into the tiling loop.  For request b and query
 * head j, with KV head h = j / (num_q_heads / num_kv_heads):
 *
 *   out[b][j][:] = softmax_pos(scale * q[b][j] . K_b[pos][h]) . V_b[pos][h]
 *
 * Computed in fp32 with an online softmax (probabilities rounded to bf16 for
 * the P.V product); out is rounded to bf16 (round-to-nearest-even).
 * A request with seq_len 0 gets out = 0.
 *
 * out          : bf16 [batch][num_q_heads][head_dim], in device memory or
 *                in page-locked host memory that the device addresses at
 *                the same pointer (cudaHostAlloc, or cudaHostRegister,
 *                under unified addressing).  In host memory the kernels
 *                store each output row across PCIe as it becomes final
 *                (zero-copy): it is complete once the stream has passed
 *                the call.  Pageable or unknown memory: PA_ERR_INVALID
 *                before any launch.  Only written, never read.
 * q            : device bf16 [batch][num_q_heads][head_dim]
 * kv_pool      : device bf16 pool (layout above); rows beyond a request's
 *                length inside its last block may hold anything (even NaN).
 * block_tables : device int32 [batch][max_blocks_per_seq]; only the first
 *                ceil(seq_len/block_size) entries of a row are read.  An
 *                entry outside [0, num_blocks) reads as a block of zeros
 *                (its positions take part with logit 0) and flags
 *                PA_DEVERR_BLOCK_ID.
 * seq_lens     : device int32 [batch]; 0 <= seq_len <= max_seq_len.  A value
 *                beyond max_blocks_per_seq*block_size is clamped and flags
 *                PA_DEVERR_SEQ_LEN.
 * max_seq_len  : host upper bound of seq_lens, used to size the split-K grid.
 * workspace    : device scratch of at least pa_decode_workspace_size() bytes
 *                (fp32 partial outputs and log-sum-exp terms of the
 *                sequence partitions), 256-byte aligned; its contents need
 *                no initialisation.
 * Schedule: batches of up to 4096 requests with at least ~4 blocks of work
 * per SM (batch * num_kv_heads * ceil(max_seq_len / block_size) >= 4 * SMs)
 * use a balanced persistent schedule -- two CTAs per SM, each taking an
 * equal contiguous share of all (request, KV head, block) units -- followed
 * by a log-sum-exp merge of the (request, head) pairs cut between CTAs.
 * Other calls use one CTA per (request, KV head, partition of up to 512
 * tokens) and the same kind of merge.
 * Supported: head_dim in {64, 128}; block_size in {16, 32}; num_q_heads a
 * multiple of num_kv_heads with group size 1..32 (above 8: the balanced
 * schedule only -- partition_tokens 0 or -1 -- and a tensor-core variant;
 * by default at head_dim 128 the tcgen05 consumer, one CTA per SM
 * streaming 128-token tiles; batches of 4097..32768 requests run on the
 * tcgen05 consumer at either head_dim, up to 4096 on either).  Others:
 * PA_ERR_UNSUPPORTED.
 * Launches: two kernels (decode + merge); the per-partition schedule skips
 * the merge when no request spans two partitions.
 * ------------------------------------------------------------------------ */
/* *num_partitions_out: CTAs of the balanced schedule, or sequence
 * partitions of the per-partition schedule (merge launched when > 1). */
int pa_decode_workspace_size(int batch, int num_q_heads, int num_kv_heads, int head_dim,
                             int block_size, int max_seq_len, size_t* bytes_out,
                             int* num_partitions_out);

int pa_decode(pa_bf16* out, const pa_bf16* q, const pa_bf16* kv_pool,
              const int32_t* block_tables, const int32_t* seq_lens, int batch,
              int num_q_heads, int num_kv_heads, int head_dim, int block_size,
              int num_blocks, int max_blocks_per_seq, int max_seq_len, float scale,
              void* workspace, size_t workspace_bytes, void* stream);

/* Kernel variant of the decode main loop. */
typedef enum pa_decode_variant {
  PA_DECODE_AUTO = 0,      /* 9..32 (token, head) columns per KV head at head_dim 128:
                              PA_DECODE_TCGEN05; otherwise PA_DECODE_MMA */
  PA_DECODE_CUDA_CORE = 1, /* fp32 FMA on CUDA cores (group 1, 2 or 4) */
  PA_DECODE_MMA = 2,       /* bf16 mma.sync with fp32 accumulate (group 1..32) */
  PA_DECODE_TCGEN05 = 3    /* tcgen05.mma into tensor memory: 128-token tiles, one issuing
                              thread, 1..32 columns (MMA N = 16 or 32); balanced schedule
                              only (size the workspace with partition_tokens = -1) */
} pa_decode_variant;

/* pa_decode with explicit choices, for measurement and tests.
 * variant          : pa_decode_variant.
 * partition_tokens : 0 = the built-in choice (see pa_decode); -1 = the
 *                    balanced schedule whatever the work (batch <= 4096,
 *                    else PA_ERR_UNSUPPORTED); > 0 = one CTA per (request,
 *                    KV head, partition of this many tokens, a multiple of
 *                    block_size).  The workspace must be sized with
 *                    pa_decode_workspace_size_ex for the same value. */
/* *balanced_out (may be NULL): 1 when the call uses the balanced schedule. */
int pa_decode_workspace_size_ex(int batch, int num_q_heads, int num_kv_heads, int head_dim,
                                int block_size, int max_seq_len, int partition_tokens,
                                size_t* bytes_out, int* num_partitions_out, int* balanced_out);

int pa_decode_ex(pa_bf16* out, const pa_bf16* q, const pa_bf16* kv_pool,
                 const int32_t* block_tables, const int32_t* seq_lens, int batch,
                 int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                 int num_blocks, int max_blocks_per_seq, int max_seq_len, float scale,
                 void* workspace, size_t workspace_bytes, int variant,
                 int partition_tokens, void* stream);

/* --------------------------------------------------------------------------
 * pa_decode_noalloc -- pa_decode for callers that cannot allocate device
 * memory.  (No counterpart on the pages: this is a packaging choice.)
 *
 * Some callers have no way to hand the library a workspace: a plugin
 * running inside a host program that owns the whole GPU memory budget and
 * forbids its own cudaMalloc calls, or a latency-critical decode loop where
 * cudaMalloc's implicit device synchronisation is not acceptable.  This
 * entry point takes the same arguments as pa_decode minus the workspace and
 * keeps the split-K partials in a fixed array compiled into the library
 * (PA_NOALLOC_SCRATCH_BYTES on every GPU that loads the library, held until
 * the process exits).  It calls no cudaMalloc/cudaFree and no allocating
 * library routine.
 *  - A call whose split-K scratch (pa_decode_workspace_size for the same
 *    arguments) exceeds PA_NOALLOC_SCRATCH_BYTES returns PA_ERR_UNSUPPORTED
 *    before launching anything; use pa_decode with a caller workspace.
 *  - The first call on each device looks up the array's device address
 *    (cudaGetSymbolAddress) with that device current; make that first call
 *    before any stream capture.
 *  - Every call on a device shares the one array and it keeps the last
 *    call's contents; nothing in it needs to start at zero.  Calls that can
 *    overlap on the GPU (different streams without ordering) race on it.
 * ------------------------------------------------------------------------ */
#define PA_NOALLOC_SCRATCH_BYTES (16u * 1024u * 1024u)

int pa_decode_noalloc(pa_bf16* out, const pa_bf16* q, const pa_bf16* kv_pool,
                      const int32_t* block_tables, const int32_t* seq_lens, int batch,
                      int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                      int num_blocks, int max_blocks_per_seq, int max_seq_len, float scale,
                      void* stream);

/* --------------------------------------------------------------------------
 * pa_decode_append -- pa_reshape_and_cache of each request's newest token,
 * then pa_decode, in one pass.
 *
 * The same results as pa_reshape_and_cache(new_k, new_v, kv_pool,
 * slot_mapping, batch, ...) followed by pa_decode(...) on the same stream,
 * for the decode step where every request has just appended one token
 * ("Paged attention in LLMs", section "The cache being stored"): request
 * b's new token is its position seq_lens[b] - 1 and slot_mapping[b] must be
 * that position's slot (block_tables[b][(L-1)/bs] * bs + (L-1) % bs, as
 * pa_alloc_append returns it); a negative slot writes nothing.  On the
 * balanced schedule there is no separate cache-write launch: the mma.sync
 * decode kernel with one warp per block puts the new row straight into the
 * staged tile and the merge kernel stores it in the pool afterwards; the
 * tcgen05 kernel, the grouped-warp and the block-pair mma.sync kernels
 * store it in the pool just before the TMA load of that block (their CTA is
 * the only one that reads those rows).  On the per-partition grid the two
 * kernels run in turn.
 * new_k, new_v : device bf16 [batch][num_kv_heads][head_dim]
 * slot_mapping : device int64 [batch]
 * Other arguments, workspace and limits as pa_decode.
 * ------------------------------------------------------------------------ */
int pa_decode_append(pa_bf16* out, const pa_bf16* q, pa_bf16* kv_pool, const pa_bf16* new_k,
                     const pa_bf16* new_v, const int64_t* slot_mapping, const int32_t* block_tables,
                     const int32_t* seq_lens, int batch, int num_q_heads, int num_kv_heads,
                     int head_dim, int block_size, int num_blocks, int max_blocks_per_seq,
                     int max_seq_len, float scale, void* workspace, size_t workspace_bytes,
                     void* stream);

/* --------------------------------------------------------------------------
 * pa_decode_multi -- several query tokens per request, causal.
 *
 * The single-token operation above, for the T newest tokens of each request
 * at once (speculative-decoding verification, chunked decode): query token
 * t of request b sits at position seq_lens[b] - T + t -- its keys and values
 * are already in the cache -- and attends to positions [0, seq_lens[b] - T
 * + t] through the block table, as in the quiz page's sketch over that
 * prefix.  A token with no position to attend to (seq_lens[b] < T - t) gets
 * out = 0.
 *
 * q, out       : bf16 [batch][T][num_q_heads][head_dim]; q in device
 *                memory, out in device or pinned host memory as for
 *                pa_decode
 * Other arguments as pa_decode.  (num_q_heads / num_kv_heads) * T <= 32.
 * Always the balanced schedule (batch <= 4096; above 8 columns up to
 * 32768 requests, on the tcgen05 consumer) and a tensor-core consumer
 * (tcgen05 for 9..32 columns at head_dim 128, mma.sync otherwise);
 * workspace from
 * pa_decode_multi_workspace_size.
 * ------------------------------------------------------------------------ */
int pa_decode_multi_workspace_size(int batch, int num_query_tokens, int num_q_heads,
                                   int num_kv_heads, int head_dim, int block_size,
                                   int max_seq_len, size_t* bytes_out);

int pa_decode_multi(pa_bf16* out, const pa_bf16* q, const pa_bf16* kv_pool,
                    const int32_t* block_tables, const int32_t* seq_lens, int batch,
                    int num_query_tokens, int num_q_heads, int num_kv_heads, int head_dim,
                    int block_size, int num_blocks, int max_blocks_per_seq, int max_seq_len,
                    float scale, void* workspace, size_t workspace_bytes, void* stream);

/* --------------------------------------------------------------------------
 * pa_decode_contiguous -- the same attention over a contiguous cache.
 *
 * The baseline paging replaces: the quiz page's comparison table, column
 * "Naive contiguous allocation" (row "Reservation per request": a buffer
 * sized for the maximum context; row "Kernel overhead": none).  Each request
 * owns one reserved run of max_len positions, keys then values:
 *
 *   kv_cache : device bf16 [batch][2][num_kv_heads][max_len][head_dim]
 *              (index 0 on the second axis keys, 1 values)
 *
 * and out[b, j] is the softmax(q K^T scale) V of pa_decode over positions
 * [0, seq_lens[b]) of that run -- no block table.  It runs pa_decode's
 * balanced kernel and arithmetic with the table lookup replaced by direct
 * 16-row tile addressing, so at equal lengths the two layouts give the same
 * result bit for bit and their timing difference is the cost of paging.
 * max_len must be a positive multiple of 16; seq_lens[b] > max_len is
 * flagged (PA_DEVERR_SEQ_LEN) and clamped.  variant: PA_DECODE_AUTO,
 * PA_DECODE_CUDA_CORE (group 1, 2, 4) or PA_DECODE_MMA.  batch <= 4096,
 * group <= 32 (above 8: mma.sync on grouped warps, as pa_decode with
 * PA_DECODE_MMA on the balanced schedule).
 * Workspace from pa_decode_contiguous_workspace_size (never 0 bytes).
 * Other arguments as pa_decode (out in device or pinned host memory).
 * ------------------------------------------------------------------------ */
int pa_decode_contiguous_workspace_size(int batch, int num_q_heads, int num_kv_heads, int head_dim,
                                        int max_len, size_t* bytes_out);

int pa_decode_contiguous(pa_bf16* out, const pa_bf16* q, const pa_bf16* kv_cache,
                         const int32_t* seq_lens, int batch, int num_q_heads, int num_kv_heads,
                         int head_dim, int max_len, float scale, void* workspace,
                         size_t workspace_bytes, int variant, void* stream);

/* Self-test of the bounded pipeline wait used by the kernels: one CTA waits
 * on a barrier phase that nothing completes, for at most limit_ns, then
 * returns.  Expect PA_DEVERR_WAIT_TIMEOUT in pa_device_error() afterwards.
 * The GPU context stays usable. */
int pa_selftest_wait_timeout(int64_t limit_ns, void* stream);

/* --------------------------------------------------------------------------
 * Host block allocator (no device memory).
 *
 * "Paged attention in LLMs": a request takes a block when it needs one and
 * another when that fills ("The fix"); a block table per request ("Keeping
 * track"); requests that share a prefix point at the same physical blocks
 * ("Sharing blocks").  Quiz page: blocks are returned as a request ends;
 * beams copy a shared block on write.
 *
 * Policy (fixed so two implementations can be compared bit for bit):
 *  - the free list is a LIFO stack; a new allocator pops blocks in
 *    `initial_order` (NULL = 0, 1, 2, ...); freed blocks are pushed on top,
 *    a request's blocks in table order;
 *  - appending into a partially filled last block whose refcount > 1 takes
 *    a fresh block, emits (src, dst), drops one reference from src and
 *    points this request at dst (copy-on-write); full blocks are never
 *    written, so never copied;
 *  - every append call is all-or-nothing: PA_ERR_OOM leaves the state as it
 *    was.
 * Not thread-safe: one handle, one thread at a time.
 * ------------------------------------------------------------------------ */
typedef struct pa_alloc pa_alloc;

int pa_alloc_create(int num_blocks, int block_size, const int32_t* initial_order,
                    pa_alloc** out);
int pa_alloc_destroy(pa_alloc* a);
int pa_alloc_add_seq(pa_alloc* a, int64_t seq_id);
/* child shares all of parent's blocks (refcount + 1 each). */
int pa_alloc_fork(pa_alloc* a, int64_t parent, int64_t child);
/* Append num_tokens tokens to one request.  slots_out (host int64
 * [num_tokens]) receives each token's slot = block*block_size + offset.
 * cow_pairs_out (host int32 [cow_cap][2]) receives (src, dst) pairs;
 * *num_cow_out their count.  cow_cap too small: PA_ERR_INVALID, no change. */
int pa_alloc_append(pa_alloc* a, int64_t seq_id, int num_tokens, int64_t* slots_out,
                    int32_t* cow_pairs_out, int cow_cap, int* num_cow_out);
/* Append tokens_each tokens to each of num_seqs requests, in the given order;
 * slots_out is [num_seqs*tokens_each] in (request, token) order. */
int pa_alloc_append_batch(pa_alloc* a, const int64_t* seq_ids, int num_seqs, int tokens_each,
                          int64_t* slots_out, int32_t* cow_pairs_out, int cow_cap,
                          int* num_cow_out);
int pa_alloc_free_seq(pa_alloc* a, int64_t seq_id);
int pa_alloc_num_free(const pa_alloc* a, int* out);
int pa_alloc_seq_len(const pa_alloc* a, int64_t seq_id, int* out);
int pa_alloc_refcount(const pa_alloc* a, int block, int* out);
/* The request's block table (host int32 [cap]); *n_out = its length. */
int pa_alloc_block_table(const pa_alloc* a, int64_t seq_id, int32_t* out, int cap, int* n_out);
/* Padded tables of several requests: tables_out host int32
 * [num_seqs][max_blocks_per_seq] (unused entries 0), seq_lens_out host int32
 * [num_seqs].  A table longer than max_blocks_per_seq: PA_ERR_INVALID. */
int pa_alloc_block_tables(const pa_alloc* a, const int64_t* seq_ids, int num_seqs,
                          int max_blocks_per_seq, int32_t* tables_out, int32_t* seq_lens_out);
/* Occupancy of the pool ("Paged attention in LLMs", sections "A worked
 * example" and "Why this helps so much": slots held vs used).
 * stats_out host int64 [5]:
 *   [0] tokens stored    = sum of the live requests' lengths
 *   [1] logical slots    = sum over live requests of table length * block_size
 *   [2] physical blocks  = blocks with refcount > 0 (shared blocks once)
 *   [3] live requests
 *   [4] free blocks
 * Internal waste = [1] - [0] (at most block_size-1 per request); slots saved
 * by sharing = [1] - [2]*block_size. */
int pa_alloc_stats(const pa_alloc* a, int64_t* stats_out);
/* Full state for comparison: free_list_out host int32 [num_blocks] gets the
 * free blocks in the order the next pops return them (*num_free_out of
 * them); refcounts_out host int32 [num_blocks]. */
int pa_alloc_dump(const pa_alloc* a, int32_t* free_list_out, int* num_free_out,
                  int32_t* refcounts_out);

#ifdef __cplusplus
}
#endif
#endif /* PA_H_ */
