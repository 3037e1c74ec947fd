/*
 * tv.h -- C ABI of libtv: PagedAttention over a block-table KV cache on B200.
 *
 * Operations, as the source pages define them:
 *   [P1] "tiny-vllm：从零构建高性能LLM推理引擎的完整指南" (zingnex.cn), secs.
 *        "PagedAttention：从操作系统借来的智慧" (fixed-size KV blocks located
 *        through a per-sequence block table), "推理流程：从Prefill到Decode"
 *        (decode appends the new token's K,V to the cache and attends over
 *        it; prefill handles the prompt tokens in parallel), "在线Softmax：
 *        数值稳定的注意力计算" (running max and correction factor), "Llama 3.2
 *        1B架构拆解" (grouped-query attention, causal mask, softmax, weighted
 *        sum of V), "BF16浮点数" (bf16 storage).
 *   [P3] "Tiny-vLLM 实战：用 C++/CUDA 手写高性能 LLM 推理引擎" (hotdry.top),
 *        secs. "内存池管理" (a page holds page_size x head_dim x num_kv_heads
 *        bf16 values; pools are preallocated, no cudaMalloc during
 *        inference), "CUDA Kernel 优化" item 3 (bf16 storage, fp32
 *        accumulation).
 *
 * Conventions shared by every call
 *   - Every pointer argument is a DEVICE pointer owned by the caller; the
 *     library allocates nothing and keeps no pointer after the call returns.
 *   - bf16 tensors are passed as void* and hold IEEE bfloat16 bit patterns.
 *   - All calls are asynchronous on `stream` (a cudaStream_t; NULL = the
 *     legacy default stream) and never synchronise the host.
 *   - Layouts (row-major, innermost last):
 *       k_pool, v_pool   [num_pages][page_size][num_kv_heads][head_dim] bf16
 *                        (slot s = page s / page_size, offset s % page_size)
 *       block_tables     [num_seqs][max_blocks_per_seq] int32: physical page
 *                        of logical block b = token positions
 *                        [b*page_size, (b+1)*page_size)
 *       context_lens     [num_seqs] int32: tokens in the cache, counting the
 *                        ones just appended
 *       q, out (decode)  [num_seqs][num_q_heads][head_dim] bf16
 *       q, out (prefill) [total_query_rows][num_q_heads][head_dim] bf16
 *   - Query head h reads KV head h / (num_q_heads / num_kv_heads).
 *   - Supported: head_dim == 64, page_size 16 or 32 ([P3] recommends 16-32
 *     tokens; the kernels stream 16-token blocks, two per 32-token page),
 *     num_q_heads a multiple of num_kv_heads with a ratio in {1, 2, 4, 8}
 *     (every call); every pointer 16-byte aligned; num_seqs
 *     <= 65535; num_pages * page_size and
 *     max_blocks_per_seq * page_size at most INT32_MAX (token positions and
 *     pool rows are 32-bit in the kernels).  Anything else returns
 *     TV_ERR_UNSUPPORTED or TV_ERR_INVALID_ARG before any launch.
 *   - `err` (nullable) is a device uint32 word; kernels OR bits into it when
 *     they meet bad data and skip that data instead of faulting:
 *       TV_DEVERR_BAD_SLOT     slot_mapping entry >= num_pages * page_size
 *       TV_DEVERR_BAD_PAGE     block-table entry outside [0, num_pages); the
 *                              page's keys are left out
 *       TV_DEVERR_BAD_CONTEXT  context_len < 0 or > max_blocks * page_size;
 *                              clamped into range
 *       TV_DEVERR_TIMEOUT      a bounded internal wait (2 s) ran out; the
 *                              affected outputs are zeros
 *       TV_DEVERR_BAD_QUERY    query_start_loc inconsistent with the context
 *       TV_DEVERR_POOL_EMPTY   the page pool had too few free pages for a
 *                              sequence (tv_pool_append_slots)
 *       TV_DEVERR_BAD_SEQ      a fork or release named a bad sequence
 *       TV_DEVERR_BAD_POSITION a RoPE position outside the cos/sin table;
 *                              that K row is written unrotated
 *   - Outputs must not alias inputs.
 *   - Return: TV_OK, or an error status; TV_ERR_CUDA means the launch failed
 *     (tv_last_cuda_error() gives the CUDA error code).
 */
#ifndef TV_H_
#define TV_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  TV_OK = 0,
  TV_ERR_INVALID_ARG = 1,
  TV_ERR_UNSUPPORTED = 2,
  TV_ERR_CUDA = 3,
  TV_ERR_SCRATCH_LIMIT = 4  /* call needs more than the library's fixed
                               scratch (tv_paged_decode_split_static) */
} tv_status;

enum {
  TV_DEVERR_BAD_SLOT = 1u << 0,
  TV_DEVERR_BAD_PAGE = 1u << 1,
  TV_DEVERR_BAD_CONTEXT = 1u << 2,
  TV_DEVERR_TIMEOUT = 1u << 3,
  TV_DEVERR_BAD_QUERY = 1u << 4,
  TV_DEVERR_POOL_EMPTY = 1u << 5,
  TV_DEVERR_BAD_SEQ = 1u << 6,
  TV_DEVERR_BAD_POSITION = 1u << 7
};

/* Human-readable name of a status. Never NULL. */
const char* tv_status_string(tv_status status);

/* The CUDA error code of the last TV_ERR_CUDA returned on this thread. */
int tv_last_cuda_error(void);

/* Library version, e.g. 100 for 0.1.0. */
int tv_version(void);

/*
 * tv_kv_append -- write token t's K row and V row into pool slot
 * slot_mapping[t] ([P1] "推理流程": append the new token's K,V to the cache;
 * [P3] "内存池管理": page layout).
 *   k_new, v_new   [num_tokens][num_kv_heads][head_dim] bf16, read only
 *   slot_mapping   [num_tokens] int32; slot = page * page_size + offset;
 *                  a negative slot is padding and is skipped; a slot beyond
 *                  the pool is skipped and flagged TV_DEVERR_BAD_SLOT
 *   k_pool, v_pool updated in place; every other byte is left unchanged
 * The copy is bit-exact.  Two tokens mapped to one slot race (either may
 * win).  num_tokens == 0 is a no-op.
 */
tv_status tv_kv_append(const void* k_new, const void* v_new,
                       const int32_t* slot_mapping, int64_t num_tokens,
                       void* k_pool, void* v_pool, int64_t num_pages,
                       int num_kv_heads, int head_dim, int page_size,
                       uint32_t* err, void* stream);

/*
 * tv_kv_append_rope -- tv_kv_append with every new K row rotated at its
 * position first ([P1] "Llama 3.2 1B架构拆解": RoPE injects the position into
 * Q and K by rotation; V is not rotated).  The pages give no pairing, angles
 * or arithmetic; this library's reading:
 *   - dimension i is rotated with i + head_dim/2 (rotate-half pairing);
 *   - rope_cos_sin  [rope_max_position][2][head_dim/2] fp32, device, 16-byte
 *                   aligned: cos (row 0) and sin (row 1) of each pair's
 *                   angle at each position (any base or scaling is the
 *                   caller's);
 *   - with x1 = k[i], x2 = k[i + head_dim/2], c, s the table entries:
 *       k'[i]            = bf16_rn(fl(fl(x1 c) - fl(x2 s)))
 *       k'[i + head_dim/2] = bf16_rn(fl(fl(x2 c) + fl(x1 s)))
 *     fl = one binary32 rounding (no fused multiply-add), bf16_rn = round
 *     to nearest even.
 *   positions   [num_tokens] int32: the token's position in its sequence; a
 *               position outside [0, rope_max_position) writes the row
 *               unrotated and flags TV_DEVERR_BAD_POSITION
 * Other arguments and behaviour as tv_kv_append.
 */
tv_status tv_kv_append_rope(const void* k_new, const void* v_new,
                            const int32_t* slot_mapping,
                            const int32_t* positions, int64_t num_tokens,
                            void* k_pool, void* v_pool, int64_t num_pages,
                            int num_kv_heads, int head_dim, int page_size,
                            const float* rope_cos_sin, int rope_max_position,
                            uint32_t* err, void* stream);

/*
 * tv_paged_decode -- one query per sequence at position context_lens[s]-1
 * attends to keys 0 .. context_lens[s]-1 of its sequence, found through the
 * block table ([P1] "PagedAttention", "推理流程", "在线Softmax", "Llama 3.2
 * 1B架构拆解"):
 *   out[s][h] = sum_j softmax_j(scale * q[s][h] . K_j) V_j
 * with fp32 accumulation and one bf16 rounding (nearest even) of the result.
 *   out            [num_seqs][num_q_heads][head_dim] bf16, written
 *   q              [num_seqs][num_q_heads][head_dim] bf16
 *   k_pool, v_pool [num_pages][page_size][num_kv_heads][head_dim] bf16
 *   block_tables   [num_seqs][max_blocks_per_seq] int32; only the first
 *                  ceil(context_lens[s] / page_size) entries are read
 *   context_lens   [num_seqs] int32; 0 gives an all-zero output row
 * Slots past a sequence's context (in its last page) are never used, so
 * they may hold anything, NaN included.
 */
tv_status tv_paged_decode(void* out, const void* q, const void* k_pool,
                          const void* v_pool, const int32_t* block_tables,
                          int max_blocks_per_seq, const int32_t* context_lens,
                          int num_seqs, int num_q_heads, int num_kv_heads,
                          int head_dim, int page_size, int64_t num_pages,
                          float scale, uint32_t* err, void* stream);

/*
 * tv_paged_decode_append -- the whole decode step in one launch: append the
 * new token of every sequence at position context_lens[s]-1 (its slot found
 * through the block table) and attend over the cache, i.e. the result of
 * tv_kv_append with slot = block_tables[s][(ctx-1)/PS]*PS + (ctx-1)%PS
 * (PS = page_size)
 * followed by tv_paged_decode ([P1] "推理流程": compute the new token's K,V,
 * append them to the cache, then attend).  The new row is written to the
 * pools and used directly from shared memory, never read back from HBM.
 *   k_new, v_new   [num_seqs][num_kv_heads][head_dim] bf16
 *   k_pool, v_pool updated in place (one row per sequence and KV head)
 *   other arguments as tv_paged_decode; context_lens[s] >= 1 counts the new
 *   token.  A sequence with context 0 appends nothing and outputs zeros.
 * The appended slot must not be read by another sequence of the same call
 * (a shared prefix page is never the page a token is appended to).
 */
tv_status tv_paged_decode_append(void* out, const void* q, const void* k_new,
                                 const void* v_new, void* k_pool, void* v_pool,
                                 const int32_t* block_tables,
                                 int max_blocks_per_seq,
                                 const int32_t* context_lens, int num_seqs,
                                 int num_q_heads, int num_kv_heads,
                                 int head_dim, int page_size,
                                 int64_t num_pages, float scale,
                                 uint32_t* err, void* stream);

/*
 * tv_paged_decode_append_rope -- tv_paged_decode_append with the new K row
 * of every sequence rotated at its position context_lens[s]-1 (the RoPE of
 * tv_kv_append_rope, same table and arithmetic) before it enters the pool
 * and the attention; q is used as given (rotated by the caller).
 */
tv_status tv_paged_decode_append_rope(
    void* out, const void* q, const void* k_new, const void* v_new,
    void* k_pool, void* v_pool, const int32_t* block_tables,
    int max_blocks_per_seq, const int32_t* context_lens, int num_seqs,
    int num_q_heads, int num_kv_heads, int head_dim, int page_size,
    int64_t num_pages, float scale, const float* rope_cos_sin,
    int rope_max_position, uint32_t* err, void* stream);

/*
 * tv_decode_workspace_size -- bytes of device workspace that
 * tv_paged_decode_balanced needs for up to num_seqs sequences on the
 * current device (it depends on the device's SM count).
 *   bytes   host pointer, written on TV_OK
 */
tv_status tv_decode_workspace_size(int num_seqs, int num_q_heads,
                                   int num_kv_heads, int head_dim,
                                   size_t* bytes);

/*
 * tv_paged_decode_balanced -- the result of tv_paged_decode (k_new == NULL)
 * or of tv_paged_decode_append (k_new, v_new given), computed by a
 * persistent grid that gives every warp the same number of K/V pages: the
 * pages of all (sequence, KV head) pairs are laid end to end and cut into
 * equal contiguous ranges.  A pair cut by range boundaries is finished from
 * per-warp partials (running max, sum and weighted V sum of each head) by
 * the log-sum-exp rule of tv_split_merge ([P1] "在线Softmax": partial
 * softmax results combine exactly through their maxima and sums); the warp
 * that writes the last partial of a pair merges them.  The source pages
 * give no schedule; this one removes the idle SMs that a grid of one CTA
 * per pair leaves when the pair count is not a multiple of the resident
 * CTA slots, and the tail that mixed context lengths cause.
 *   workspace        device memory of at least tv_decode_workspace_size()
 *                    bytes, 16-byte aligned, ZERO-FILLED before its first
 *                    use; each call leaves it zero-filled again unless a
 *                    bounded wait ran out (TV_DEVERR_TIMEOUT), after which
 *                    it must be zero-filled again
 *   workspace_bytes  its size; too small returns TV_ERR_INVALID_ARG
 *   other arguments as tv_paged_decode / tv_paged_decode_append.
 * Calls that overlap on the GPU (unordered streams) need separate
 * workspaces.  Above 512 sequences, with max_blocks_per_seq >= 2^24 or
 * num_pages >= 2^26 - 1, or when num_seqs * num_kv_heads *
 * max_blocks_per_seq reaches 2^31, the call runs the one-CTA-per-pair
 * kernel of tv_paged_decode instead and leaves the workspace untouched.
 * Results equal tv_paged_decode's up to fp32 summation order.
 */
tv_status tv_paged_decode_balanced(void* out, const void* q,
                                   const void* k_new, const void* v_new,
                                   void* k_pool, void* v_pool,
                                   const int32_t* block_tables,
                                   int max_blocks_per_seq,
                                   const int32_t* context_lens, int num_seqs,
                                   int num_q_heads, int num_kv_heads,
                                   int head_dim, int page_size,
                                   int64_t num_pages, float scale,
                                   void* workspace, size_t workspace_bytes,
                                   uint32_t* err, void* stream);

/*
 * tv_paged_decode_split -- tv_paged_decode restricted to logical key
 * partitions p = [p*partition_tokens, (p+1)*partition_tokens) of each
 * context (the blockwise online softmax of [P1] "在线Softmax"):
 *   partial_out  [num_seqs][num_q_heads][max_partitions][head_dim] fp32:
 *                the normalised attention over partition p alone
 *   partial_lse  [num_seqs][num_q_heads][max_partitions] fp32: natural
 *                log of sum_j exp(scale * q.K_j) over partition p
 * An empty partition (p >= ceil(context / partition_tokens)) gets
 * partial_out = 0 and partial_lse = -infinity.  partition_tokens must be a
 * positive multiple of page_size; max_partitions >= the largest
 * ceil(context_lens[s] / partition_tokens) the caller expects (partitions
 * beyond max_partitions are not computed).
 */
tv_status tv_paged_decode_split(float* partial_out, float* partial_lse,
                                const void* q, const void* k_pool,
                                const void* v_pool,
                                const int32_t* block_tables,
                                int max_blocks_per_seq,
                                const int32_t* context_lens, int num_seqs,
                                int num_q_heads, int num_kv_heads,
                                int head_dim, int page_size,
                                int64_t num_pages, float scale,
                                int partition_tokens, int max_partitions,
                                uint32_t* err, void* stream);

/*
 * tv_split_merge -- combine the partials of tv_paged_decode_split:
 *   M = max_p lse_p over p < min(ceil(context/partition_tokens),
 *   max_partitions);  out = sum_p e^(lse_p - M) o_p / sum_p e^(lse_p - M)
 *   out          [num_seqs][num_q_heads][head_dim] bf16, written
 *   partial_out, partial_lse as written by tv_paged_decode_split
 * A sequence with no keys gets a zero row.
 */
tv_status tv_split_merge(void* out, const float* partial_out,
                         const float* partial_lse,
                         const int32_t* context_lens, int num_seqs,
                         int num_q_heads, int head_dim, int partition_tokens,
                         int max_partitions, void* stream);

/*
 * tv_paged_prefill -- chunked prefill over the paged cache ([P1] "推理流程":
 * prefill processes the prompt tokens in parallel under a causal mask).
 * Sequence s owns query rows [query_start_loc[s], query_start_loc[s+1]);
 * their K,V must already be in the cache (tv_kv_append).  With T_s rows and
 * C = context_lens[s], row i sits at position C - T_s + i and attends to
 * keys 0 .. C - T_s + i.  QK^T and PV run on the tcgen05 tensor cores (bf16
 * in, fp32 accumulate in tensor memory); P enters PV as the sum of two bf16
 * terms (p rounded, plus the rounding remainder).
 *   out              [total_rows][num_q_heads][head_dim] bf16, written
 *   q                [total_rows][num_q_heads][head_dim] bf16
 *   num_query_rows   total_rows (the row count of q and out)
 *   query_start_loc  [num_seqs + 1] int32, non-decreasing, [0] == 0,
 *                    [num_seqs] <= num_query_rows
 *   max_query_len    >= every T_s (sizes the grid); rows beyond a
 *                    sequence's T_s are not touched; at most 65535 blocks
 *                    of 256 / G rows (G = num_q_heads / num_kv_heads)
 *   workspace        NULL, or device memory of at least
 *                    tv_prefill_workspace_size() bytes, 16-byte aligned, no
 *                    initial contents needed; too small or misaligned
 *                    returns TV_ERR_INVALID_ARG.  Given, a one-CTA kernel
 *                    first lists the work blocks (256 / G query rows of
 *                    one sequence) by their number of key tiles, costliest
 *                    first, and the attention grid runs them in that order,
 *                    so that long-context blocks do not start last and hold
 *                    a few SMs while the rest idle.  The results are the
 *                    same with and without it.  Concurrent calls need
 *                    separate workspaces.
 *   workspace_bytes  its size
 * A sequence with T_s > C is flagged TV_DEVERR_BAD_QUERY and skipped.
 * Supported: num_q_heads == G * num_kv_heads with G = 1, 2, 4 or 8 (one MMA
 * tile = 128 / G query rows x the G heads of a KV head; TV_ERR_UNSUPPORTED
 * otherwise) and scale > 0 (TV_ERR_INVALID_ARG otherwise: the kernel takes
 * each key tile's maximum on the raw scores q.K and scales it afterwards,
 * which equals the maximum of the scaled scores only for a positive scale).
 */
tv_status tv_paged_prefill(void* out, const void* q, int64_t num_query_rows,
                           const int32_t* query_start_loc, const void* k_pool,
                           const void* v_pool, const int32_t* block_tables,
                           int max_blocks_per_seq, const int32_t* context_lens,
                           int num_seqs, int max_query_len, int num_q_heads,
                           int num_kv_heads, int head_dim, int page_size,
                           int64_t num_pages, float scale, void* workspace,
                           size_t workspace_bytes, uint32_t* err,
                           void* stream);

/*
 * tv_prefill_workspace_size -- bytes of the optional tv_paged_prefill
 * workspace for num_seqs sequences and the given max_query_len (4 bytes per
 * 32-row block of every sequence, rounded up to 16: enough for every group
 * size; a call checks the size its own group needs, 4 bytes per block of
 * 256 / G rows).
 *   bytes   host pointer, written on TV_OK
 */
tv_status tv_prefill_workspace_size(int num_seqs, int max_query_len,
                                    size_t* bytes);

/*
 * tv_paged_decode_split_static -- tv_paged_decode_split followed by
 * tv_split_merge in one call that allocates nothing: the fp32 partials go to
 * a fixed array inside the library instead of caller buffers.  The source
 * pages have no counterpart of this call; it exists for callers that cannot
 * allocate on the decode path: engines that give (almost) all device memory
 * to the KV page pool at start-up and allow no allocation while serving,
 * step loops that cannot afford cudaMalloc/cudaFree (which may block and
 * synchronise the device), and plain C hosts with no device allocator.
 *   out and every other argument: as tv_paged_decode_split / tv_split_merge;
 *   out [num_seqs][num_q_heads][head_dim] bf16 receives the merged result.
 * Limits and sharing:
 *   - the array holds TV_STATIC_SCRATCH_FLOATS floats (32 MiB) per device
 *     and stays allocated on every GPU that loads the library until exit;
 *   - a call needs num_seqs * num_q_heads * max_partitions * (head_dim + 1)
 *     floats; a larger one returns TV_ERR_SCRATCH_LIMIT before any launch;
 *   - every call on a device shares the array, which keeps the last call's
 *     contents (nothing in it needs to start at zero: each call rewrites
 *     every partial it reads); calls that overlap on the GPU (unordered
 *     streams) race on it;
 *   - the first call on a device looks up the array's device address with
 *     that device current; make that first call before any stream capture.
 *     The address is kept per device together with the id of the CUDA
 *     context it belongs to; when a later call finds another context
 *     current (e.g. after cudaDeviceReset) it looks the address up again,
 *     so that first call in the new context should also come before any
 *     capture.
 * Returns TV_ERR_CUDA when that lookup fails.
 */
#define TV_STATIC_SCRATCH_FLOATS (1 << 23)

tv_status tv_paged_decode_split_static(
    void* out, const void* q, const void* k_pool, const void* v_pool,
    const int32_t* block_tables, int max_blocks_per_seq,
    const int32_t* context_lens, int num_seqs, int num_q_heads,
    int num_kv_heads, int head_dim, int page_size, int64_t num_pages,
    float scale, int partition_tokens, int max_partitions, uint32_t* err,
    void* stream);

/*
 * tv_selftest_wait_timeout -- exercises the bounded wait behind every
 * TV_DEVERR_TIMEOUT: one thread waits on an mbarrier that nothing completes,
 * gives up after limit_ns nanoseconds of %globaltimer (clamped to the
 * library's 2 s), ORs TV_DEVERR_TIMEOUT into *err and returns.  The call
 * faults nothing and leaves the context usable; it is how the failure path
 * is tested without a failure.  The pages have no counterpart.
 *   err        device uint32 word (required)
 *   waited_ns  device uint64 (nullable): time actually waited
 */
tv_status tv_selftest_wait_timeout(uint32_t* err, int64_t limit_ns,
                                   uint64_t* waited_ns, void* stream);

/*
 * ---- Device page pool -------------------------------------------------------
 * The KV pages of [P3] "内存池管理" as a device-resident pool: a free-page stack
 * and a reference count per page, so that a decode step -- room for the new
 * token, then tv_paged_decode_append -- needs no host round trip and can be
 * captured in a CUDA graph.  Pages are allocated on demand, returned when a
 * sequence is released, and shared between sequences by tv_pool_fork (prefix
 * sharing); a shared page is copied before it is written ([P1]
 * "PagedAttention": copy-on-write).  The pages give no free-list layout, no
 * order of allocation and no sharing rule beyond these; the rules below are
 * this library's, chosen so every call is deterministic.
 *
 * pool_state: device int32 array of TV_POOL_STATE_INTS(num_pages) entries,
 * caller-owned, set up by tv_pool_init and changed only by the tv_pool_*
 * calls:
 *   [0] number of free pages (top of the stack)   [2] slots written by the
 *   last tv_pool_append_slots   [3] page size   [4 .. 4+NP) free-page stack
 *   (pop takes entry top-1)   then NP reference counts, 2 x NP scratch
 *   words (zero between calls) and TV_POOL_MAX_SEQS growth marks: entry s
 *   is 1 when the last tv_pool_append_slots gave sequence s its tokens, 0
 *   when it did not (no tokens asked, pool exhausted, or a flagged error);
 *   entries at and beyond that call's num_seqs are left as they were.
 * A page's reference count is the number of block-table rows holding it.
 * Every pool call serves at most TV_POOL_MAX_SEQS sequences
 * (TV_ERR_UNSUPPORTED above), runs as one CTA, and is ordered with the
 * caller's other work by `stream`.
 */
#define TV_POOL_MAX_SEQS 1024
#define TV_POOL_STATE_INTS(num_pages) \
  (4 + 4 * (int64_t)(num_pages) + TV_POOL_MAX_SEQS)

/*
 * tv_pool_init -- every page free, except those the first
 * ceil(context_lens[s] / page_size) entries of each block-table row hold
 * (counted); the free pages are stacked in descending id order, so a fresh
 * pool hands out pages 0, 1, 2, ...  block_tables may be NULL (an empty
 * pool).  page_size (16 or 32) is kept in the state; every later pool call
 * on it uses it (tv_pool_append_slots with another page_size flags
 * TV_DEVERR_BAD_SEQ and changes nothing).
 */
tv_status tv_pool_init(int32_t* pool_state, int64_t num_pages, int page_size,
                       const int32_t* block_tables, int max_blocks_per_seq,
                       const int32_t* context_lens, int num_seqs,
                       uint32_t* err, void* stream);

/*
 * tv_pool_append_slots -- room for num_new_tokens[s] tokens at positions
 * context_lens[s] .. context_lens[s] + n - 1 of every sequence, in batch
 * order:
 *   - if the partly filled page those positions start in is shared (count
 *     > 1), the sequence first takes a fresh page and copies that page's K
 *     and V into it (copy-on-write), unless every holder of the page writes
 *     into it in this call and this sequence is the last of them in batch
 *     order (it keeps the page);
 *   - then it takes one fresh page per page boundary crossed;
 *   - needs are reserved in batch order and served all-or-nothing: once a
 *     sequence cannot be served, no later one is (TV_DEVERR_POOL_EMPTY; those
 *     sequences are left unchanged);
 *   - context_lens[s] += n for every served sequence.
 *   num_new_tokens  [num_seqs] int32, or NULL: one token for every sequence
 *                   with context_lens[s] > 0 (a decode step)
 *   slot_mapping    NULL, or room for the sum of n: receives the slots of the
 *                   new tokens of the served sequences in batch order (as
 *                   tv_kv_append takes them); their count is pool_state[2]
 *   k_pool, v_pool  the pools (copy-on-write copies whole pages)
 */
tv_status tv_pool_append_slots(int32_t* pool_state, int64_t num_pages,
                               int32_t* block_tables, int max_blocks_per_seq,
                               int32_t* context_lens,
                               const int32_t* num_new_tokens, int num_seqs,
                               int32_t* slot_mapping, void* k_pool,
                               void* v_pool, int num_kv_heads, int head_dim,
                               int page_size, uint32_t* err, void* stream);

/*
 * tv_pool_fork -- for i = 0 .. num_pairs-1 in order: the empty sequence
 * dst_seqs[i] (context 0) takes the block-table entries and context of
 * src_seqs[i]; each shared page's count grows by one.  A pair whose
 * destination is not empty, or that names a bad index, is skipped and
 * flagged TV_DEVERR_BAD_SEQ.  src_seqs, dst_seqs: device int32 arrays.
 */
tv_status tv_pool_fork(int32_t* pool_state, int64_t num_pages,
                       int32_t* block_tables, int max_blocks_per_seq,
                       int32_t* context_lens, int num_seqs,
                       const int32_t* src_seqs, const int32_t* dst_seqs,
                       int num_pairs, uint32_t* err, void* stream);

/*
 * tv_pool_release -- for each listed sequence (device int32 array, in
 * order) every page reference is dropped, its row becomes -1 and its
 * context 0; pages whose count reaches zero go back on the stack in
 * ascending id order (so the largest of them is handed out first).
 */
tv_status tv_pool_release(int32_t* pool_state, int64_t num_pages,
                          int32_t* block_tables, int max_blocks_per_seq,
                          int32_t* context_lens, int num_seqs,
                          const int32_t* seqs, int num_release, uint32_t* err,
                          void* stream);

/*
 * tv_decode_step -- one decode step of every live sequence, device-side
 * only: tv_pool_append_slots with num_new_tokens = NULL, then
 * tv_paged_decode_append (the new token's K/V go to position ctx-1 of the
 * grown context; out = attention of q over it), or, when workspace is not
 * NULL, tv_paged_decode_balanced with k_new / v_new and that workspace (for
 * batches of mixed lengths).  Only the sequences whose context the slot
 * reservation grew (growth mark 1 in pool_state) append and attend; every
 * other sequence is idle for this step: it appends nothing, its output row
 * is zeros and its pages are left untouched.  That covers context 0, a
 * sequence left unserved by an exhausted pool (TV_DEVERR_POOL_EMPTY; it
 * keeps its context and every cached row, and can be stepped again once
 * pages are released) and one flagged TV_DEVERR_BAD_CONTEXT (full) or
 * TV_DEVERR_BAD_PAGE.  Two launches, no host synchronisation, so a run of
 * steps can be captured in one CUDA graph.  Arguments as
 * tv_pool_append_slots and tv_paged_decode_append.
 */
tv_status tv_decode_step(int32_t* pool_state, int64_t num_pages, void* out,
                         const void* q, const void* k_new, const void* v_new,
                         void* k_pool, void* v_pool, int32_t* block_tables,
                         int max_blocks_per_seq, int32_t* context_lens,
                         int num_seqs, int num_q_heads, int num_kv_heads,
                         int head_dim, int page_size, float scale,
                         void* workspace, size_t workspace_bytes,
                         uint32_t* err, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* TV_H_ */
