/*
 * pkv.h - C ABI of the paged KV-cache decode library (sm_100a).
 *
 * Operations on a KV cache split into fixed-size blocks that sit
 * non-contiguously in one physical pool per K and V:
 *
 *   paged_attn_decode  single-query attention of every sequence over its
 *                      cached tokens, read through its block table
 *   kv_cache_append    scatter new tokens' K/V into their pool slots
 *   kv_block_copy      whole-block copies (copy-on-write of shared blocks)
 *   kv_block_swap      whole-block copies between the device pools and a swap
 *                      space in page-locked host memory
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Pointers. Every data pointer is a DEVICE pointer owned by the caller, with
 * two exceptions. The `out` of the decode entry points, and the four pools of
 * kv_block_swap, may also be page-locked host memory that the device
 * addresses directly (unified addressing, e.g. from cudaHostAlloc). The
 * kernels then move the data over the bus with plain loads and stores, and
 * no separate copy is needed; the caller reads a result once the stream has
 * passed the call. The library never allocates,
 * frees or retains memory. Block allocation is host
 * bookkeeping over integer block ids, and needs no device allocation during
 * generation (page "추론 엔진에서의 메모리 가상화", molayo1419.me, block
 * manager section).
 *
 * Streams. `stream` is a cudaStream_t passed as void*; NULL means the legacy
 * default stream. Work is enqueued on it and the call returns without
 * synchronising.
 *
 * Element types. pkv_dtype gives the element type of q, out and both pools.
 *
 * Pool layout. Both pools are [num_blocks][num_kv_heads][block_size][head_dim],
 * row-major, head_dim contiguous. Token t of a sequence with block table bt
 * is at block bt[t / block_size], slot t % block_size. One (block, kv head)
 * slice is block_size*head_dim contiguous elements.
 *
 * Errors. Argument errors that the host can check return PKV_EINVAL or
 * PKV_EUNSUPPORTED synchronously, with nothing enqueued. A failed launch
 * returns PKV_ECUDA. Conditions only the device can see (a block id outside
 * [0, num_blocks), a slot beyond the pool, a context length above
 * max_context_len) never fault. The offending access is skipped (its tokens
 * are masked), and if `err` is non-NULL the first such condition's
 * PKV_DEV_* code is stored there with an atomic compare-and-swap from 0.
 * The caller zeroes *err and reads it after the stream completes.
 */
#ifndef PKV_H_
#define PKV_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  PKV_OK = 0,
  PKV_EINVAL = -1,       /* bad argument (null pointer, negative size, misalignment...) */
  PKV_EUNSUPPORTED = -2, /* valid but not implemented (head_dim, block_size, group size) */
  PKV_ECUDA = -3,        /* a CUDA runtime call or launch failed */
} pkv_status;

typedef enum { PKV_F32 = 0, PKV_F16 = 1, PKV_BF16 = 2 } pkv_dtype;

/* Device-side error codes stored into *err (first one wins). */
enum {
  PKV_DEV_BAD_BLOCK = 1,     /* block-table entry outside [0, num_blocks) */
  PKV_DEV_BAD_SLOT = 2,      /* append slot >= num_blocks * block_size */
  PKV_DEV_BAD_PAIR = 3,      /* copy or swap pair with a block id outside its pool */
  PKV_DEV_CONTEXT_LEN = 4,   /* context_lens[s] > max_context_len or > table capacity */
  PKV_DEV_WAIT_TIMEOUT = 5,  /* an on-chip copy wait gave up (never expected) */
};

/*
 * Bytes of device workspace paged_attn_decode needs for these sizes: a few
 * scheduling words, the work list (one 8-byte entry per possible
 * (sequence, partition) pair) and two int32 per sequence for the
 * shared-prefix grouping, plus, when a context can span several
 * partitions, merge counters and one fp32 output row and one fp32
 * log-sum-exp per (sequence, query head, partition), and last the
 * tail-split pieces: min(512, num_seqs * num_heads * partitions) of them,
 * each a counter and 8 fp32 rows of head_dim with their log-sum-exp values
 * (about 2 MB at head_dim 128). Always > 0 for num_seqs > 0. This function
 * is pure arithmetic: it does not touch the GPU.
 */
size_t pkv_decode_workspace_bytes(int num_seqs, int num_heads, int head_dim,
                                  int max_context_len, int partition_size);

/*
 * partition_size value that lets the library choose the partition length from
 * the batch shape (see pkv_resolve_partition). Accepted by every decode call
 * and by pkv_decode_workspace_bytes, which resolve it the same way.
 */
#define PKV_PARTITION_AUTO (-1)

/*
 * The partition length a decode call uses for partition_size.
 *
 * Splitting a context into partitions (page "PagedAttention Analysis",
 * section 3: attention over any split of the tokens recombines exactly by
 * log-sum-exp weights) is what lets a small batch of long contexts spread over
 * all SMs. PKV_PARTITION_AUTO asks for about 1024 (sequence, partition, query
 * head) rows in total, i.e. about one wave of work items at 4 query heads per
 * KV head: with L = max(max_context_len, 1) and
 * n = ceil(1024 / (num_seqs * num_heads)), it returns ceil(L / n) rounded up to
 * a multiple of 16 and clamped to [256, 2048]. A batch of 32 or more sequences
 * of 32 heads therefore gets 2048-token partitions, and one sequence of 4096
 * tokens gets 256-token ones. Any other partition_size is returned unchanged.
 * Pure arithmetic: it does not touch the GPU.
 */
int pkv_resolve_partition(int num_seqs, int num_heads, int max_context_len, int partition_size);

/*
 * Decode kernel selection for fp16 / bf16 (a process-wide setting, for tuning
 * and tests; the results agree within the accuracy bound either way).
 *
 * Two kernels implement paged_attn_decode and paged_attn_decode_append:
 *   - the persistent kernel: a one-CTA plan launch builds a work list from
 *     context_lens, then two CTAs per SM pull (sequence, partition, KV head)
 *     items, merging split contexts through the workspace. It balances large
 *     and ragged batches. With one or two query heads per KV head, when the
 *     last items would leave more than half of the CTAs idle, each of them is
 *     attended as up to 8 pieces and merged the same way.
 *   - the single-wave kernel: when every (sequence, KV head, partition) of
 *     the call fits in one wave of CTAs, one launch with no plan. CTA
 *     (p, h, s) attends partition p, and the partitions of one (sequence, KV
 *     head) form a thread-block cluster (at most 16) whose first CTA merges
 *     them through distributed shared memory. Contexts of at most 64 tokens
 *     are attended one warp per (sequence, KV head). The workspace is not
 *     touched (it is still validated) except by the split form below, and
 *     shared-prefix grouping does not apply. Under PKV_PARTITION_AUTO this kernel chooses its own partition
 *     length: the most partitions (of at least 64 tokens, at most 16) that
 *     keep the call within one wave.
 *
 * A single-wave CTA has 4 warps, or 8 when the call has at most one CTA per
 * SM and every warp gets at least two 16-token tiles (so that each SM
 * sub-partition still runs two warps). Under PKV_PARTITION_AUTO, a few very
 * long contexts (tens of thousands of tokens on a handful of (sequence, KV
 * head) pairs) are spread over several clusters of 8 CTAs per pair: each
 * cluster merges its partitions into a workspace slot, and a second launch
 * merges the slots into out. The workspace is then used (its partition
 * slots), as by the persistent kernel.
 *
 * PKV_DISPATCH_AUTO (the default) takes the single-wave kernel whenever the
 * call fits it and no warp gets more than 64 16-token tiles, else the
 * persistent one. (The single-wave kernel fixes one CTA per partition. Only
 * max_context_len is known on the host, so one long sequence among short ones
 * would run on a few CTAs there, while the persistent kernel spreads it.) PKV_DISPATCH_PERSISTENT always takes
 * the persistent kernel. PKV_DISPATCH_WAVE_CTA never uses the warp-per-item
 * form and keeps CTAs at 4 warps; PKV_DISPATCH_WAVE_CTA8 never uses the
 * warp-per-item form and takes 8-warp CTAs whenever they fit one per SM.
 * PKV_DISPATCH_WAVE_WARP uses the warp-per-item form for any call with one
 * partition (partition_size 0, AUTO, or >= the longest context), and
 * otherwise the persistent kernel.
 *
 * Returns the previous mode, or PKV_EINVAL for an unknown mode (the setting
 * is then unchanged). Safe to call from any thread; calls already issued are
 * unaffected.
 */
#define PKV_DISPATCH_AUTO 0
#define PKV_DISPATCH_PERSISTENT 1
#define PKV_DISPATCH_WAVE_CTA 2
#define PKV_DISPATCH_WAVE_WARP 3
#define PKV_DISPATCH_WAVE_CTA8 4
int pkv_set_decode_dispatch(int mode);

/*
 * paged_attn_decode - one decode step of attention over a paged KV cache.
 *
 * For every sequence s and query head h, with G = num_heads / num_kv_heads,
 * g = h / G and L = context_lens[s]:
 *   o[s][h] = sum_{t<L} softmax_t(scale * q[s][h] . k_t) * v_t
 * where k_t and v_t are token t's vectors of KV head g, found through
 * block_tables[s]. This is the causal attention of the newest token over all
 * L cached tokens, which includes itself (page "PagedAttention", newikis,
 * section "Mathematical formulation": causal attention, and its block-wise
 * form, which is identical in value). Scores are taken block by block with a
 * running max and sum. That is the online-softmax walk over the block table
 * in page "PagedAttention Analysis" (ryotta.opik.net), section 3.
 * Accumulation is fp32. The output is rounded to the input type
 * (round-to-nearest-even).
 *
 * Long contexts are split into partitions of partition_size tokens. Each
 * partition is attended independently, and the partials are combined by
 * log-sum-exp weights.
 *
 * Sequences next to each other in the batch whose block tables start with the
 * same physical blocks (forked samples, beams, cached prefixes: page
 * "PagedAttention Analysis", section 4) are attended together when
 * num_heads / num_kv_heads is 1 or 2: the whole 16-token tiles of their common
 * leading blocks are read once for all of them. Each sequence still gets its
 * own attention over its own tokens; only the fp32 summation order differs.
 * (Calls small enough for the single-wave kernel, see pkv_set_decode_dispatch,
 * attend every sequence alone.)
 *
 * out            [num_seqs][num_heads][head_dim], written entirely. A sequence
 *                with L <= 0 gets zeros. Device memory, or page-locked host
 *                memory the device can address (see Pointers).
 * q              [num_seqs][num_heads][head_dim]
 * k_pool, v_pool [num_blocks][num_kv_heads][block_size][head_dim]. Must be
 *                16-byte aligned.
 * block_tables   int32 [num_seqs][max_blocks_per_seq], physical block ids.
 *                Entries at or beyond ceil(L / block_size) are never read.
 * context_lens   int32 [num_seqs]. Precondition: 0 <= L <= max_context_len,
 *                and ceil(L / block_size) <= max_blocks_per_seq.
 * max_context_len a host-side upper bound on context_lens. It sizes the
 *                grid and the workspace, so the call needs no device-to-host read.
 * scale          score multiplier; 1/sqrt(head_dim) gives the usual attention.
 * partition_size tokens per partition. 0 means no split (one partition of
 *                the whole context), PKV_PARTITION_AUTO lets the library
 *                choose (pkv_resolve_partition for the persistent kernel; see
 *                pkv_set_decode_dispatch for the single-wave one). Otherwise
 *                a positive multiple of 16.
 * workspace      device scratch of at least pkv_decode_workspace_bytes(...)
 *                bytes, 256-byte aligned. Its contents on entry do not
 *                matter. Calls that overlap in time must not share it.
 * err            nullable device int32 error word (see above).
 *
 * Supported: head_dim in {64, 128}; f32 with any block_size >= 1; f16/bf16
 * with block_size a multiple of 8 (up to 256) and num_heads/num_kv_heads <= 8.
 * A block id outside [0, num_blocks) masks the tokens of its 16-token tile
 * (with block_size 8 or another odd multiple of 8, a tile spans two blocks).
 * Anything else returns PKV_EUNSUPPORTED.
 */
int paged_attn_decode(void *out, const void *q, const void *k_pool, const void *v_pool,
                      const int32_t *block_tables, const int32_t *context_lens, int num_seqs,
                      int num_heads, int num_kv_heads, int head_dim, int block_size,
                      int max_blocks_per_seq, int num_blocks, int max_context_len, float scale,
                      int dtype, int partition_size, void *workspace, size_t workspace_bytes,
                      int32_t *err, void *stream);

/* Size of the library-owned scratch array used by paged_attn_decode_static_ws. */
#define PKV_STATIC_WS_BYTES (64u * 1024u * 1024u)

/*
 * paged_attn_decode_static_ws - paged_attn_decode for callers that cannot
 * allocate device memory when they decode. The pages describe nothing like
 * it; it is a convenience of this library.
 *
 * Who needs it: a serving engine that reserved (almost) all device memory for
 * its KV block pool at start-up, where a later cudaMalloc for split-context
 * workspace may fail or bypass the engine's allocator. Also hosts that allow
 * no device allocation after initialisation, because cudaMalloc can
 * synchronise the device and takes an unpredictable time.
 *
 * Arguments and results are those of paged_attn_decode, without workspace and
 * workspace_bytes. The workspace instead comes from a fixed array of
 * PKV_STATIC_WS_BYTES (64 MiB) inside the library. This call allocates
 * nothing itself: no cudaMalloc, cudaFree or allocating library call.
 *
 * Limits and sharing:
 *  - If pkv_decode_workspace_bytes(...) for the arguments exceeds
 *    PKV_STATIC_WS_BYTES, the call returns PKV_EUNSUPPORTED and enqueues
 *    nothing; use paged_attn_decode with your own workspace then.
 *  - Each GPU holds its own copy of the array from the first call made on it
 *    until the process exits.
 *  - The first call on a device looks up that copy's address (one
 *    cudaGetSymbolAddress) with the device current. Make that first call
 *    before any stream capture. The address is kept per device together
 *    with the id of the context it belongs to; after a cudaDeviceReset the
 *    next call sees a new context and looks the address up again.
 *  - num_seqs <= 0 needs no workspace: the call then returns what
 *    paged_attn_decode returns for the same arguments.
 *  - All calls on a device share the one array and it keeps the last call's
 *    contents; the decode resets what it needs on every call. Calls whose
 *    GPU work can overlap in time (different streams without ordering between
 *    them) race on the array and give wrong results; order them.
 */
int paged_attn_decode_static_ws(void *out, const void *q, const void *k_pool, const void *v_pool,
                                const int32_t *block_tables, const int32_t *context_lens,
                                int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                                int block_size, int max_blocks_per_seq, int num_blocks,
                                int max_context_len, float scale, int dtype, int partition_size,
                                int32_t *err, void *stream);

/*
 * paged_attn_decode_append - one decode step with the cache-append fused in.
 *
 * For every sequence s with L = context_lens[s] >= 1 and every KV head h,
 * token L-1 is the newest token: its K/V rows k_new[s][h][:] and
 * v_new[s][h][:] are written into its pool slot (block
 * block_tables[s][(L-1) / block_size], slot (L-1) % block_size). The decode is
 * then paged_attn_decode over all L tokens, taking the newest one from
 * k_new / v_new. The result equals kv_cache_append with
 * slot_mapping[s] = block_tables[s][(L-1)/B]*B + (L-1)%B followed by
 * paged_attn_decode, in one pass: the new rows travel with the sequence's
 * work, so no separate append launch is needed. Page "PagedAttention Analysis"
 * (ryotta.opik.net), section 3, notes that vLLM fuses its kernels to soften
 * the cost of the block-table indirection.
 *
 * k_new, v_new  [num_seqs][num_kv_heads][head_dim], 16-byte aligned.
 * k_pool, v_pool are written, at exactly those slots.
 * Other arguments, errors and the workspace are those of paged_attn_decode.
 * fp16 / bf16 only (PKV_EUNSUPPORTED for f32). Precondition: the last block
 * of each sequence is its own. That holds after copy-on-write, which makes a
 * shared block private before the first write into it.
 */
int paged_attn_decode_append(void *out, const void *q, const void *k_new, const void *v_new,
                             void *k_pool, void *v_pool, const int32_t *block_tables,
                             const int32_t *context_lens, int num_seqs, int num_heads,
                             int num_kv_heads, int head_dim, int block_size,
                             int max_blocks_per_seq, int num_blocks, int max_context_len,
                             float scale, int dtype, int partition_size, void *workspace,
                             size_t workspace_bytes, int32_t *err, void *stream);

/*
 * kv_cache_append - write new tokens' K/V into their slots.
 *
 * For each token i < num_tokens with slot = slot_mapping[i] >= 0 and every KV
 * head h:
 *   k_pool[slot / block_size][h][slot % block_size][:] = k_new[i][h][:]
 *   v_pool[slot / block_size][h][slot % block_size][:] = v_new[i][h][:]
 * A new token goes into the free slot of its sequence's last block (page
 * "PagedAttention 논문 쉽게 읽기", iplexlaw.co.kr, section 2). Negative slots are
 * skipped. A slot >= num_blocks*block_size is skipped and reported in *err.
 * The copy is bit-exact.
 *
 * k_new, v_new  [num_tokens][num_kv_heads][head_dim], 16-byte aligned.
 * slot_mapping  int64 [num_tokens]. Precondition: the non-negative slots are
 *               distinct. Otherwise which token lands in a repeated slot is
 *               unspecified.
 */
int kv_cache_append(void *k_pool, void *v_pool, const void *k_new, const void *v_new,
                    const int64_t *slot_mapping, int num_tokens, int num_kv_heads,
                    int head_dim, int block_size, int num_blocks, int dtype, int32_t *err,
                    void *stream);

/*
 * kv_block_copy - copy whole physical blocks, as copy-on-write requires.
 *
 * For each pair i < num_pairs, (src, dst) = (src_dst[2i], src_dst[2i+1]), all
 * num_kv_heads*block_size*head_dim elements of block src are copied to block
 * dst, in both pools. A write into a block whose refcount is above one copies
 * the block first (page "추론 엔진에서의 메모리 가상화", molayo1419.me,
 * copy-on-write section: old block #11 copied into new block #45). The copy
 * is bit-exact.
 *
 * src_dst  device int32 [num_pairs][2]. Precondition: the dst blocks are
 *          distinct, and no dst is also a src in the same call. Pairs run
 *          concurrently. A pair with an id outside [0, num_blocks) is
 *          skipped and reported in *err.
 */
int kv_block_copy(void *k_pool, void *v_pool, const int32_t *src_dst, int num_pairs,
                  int num_kv_heads, int head_dim, int block_size, int num_blocks, int dtype,
                  int32_t *err, void *stream);

/*
 * kv_block_swap - copy whole blocks between two pools of the same block shape:
 * the device pools and a swap space in page-locked host memory, in either
 * direction.
 *
 * For each pair i < num_pairs, (src, dst) = (src_dst[2i], src_dst[2i+1]), all
 * num_kv_heads*block_size*head_dim elements of block src of (src_k, src_v)
 * are copied to block dst of (dst_k, dst_v). This is the data half of
 * swapping (page "PagedAttention Analysis", ryotta.opik.net, section 6): when
 * memory runs short, the blocks of a preempted sequence are copied to CPU
 * memory, which has its own block allocator, all of a sequence's blocks
 * together; they are copied back when it resumes. The copy is bit-exact.
 *
 * dst_k, dst_v  [dst_blocks][num_kv_heads][block_size][head_dim]
 * src_k, src_v  [src_blocks][num_kv_heads][block_size][head_dim]
 *               Each of the four may be device memory or page-locked host
 *               memory that the device addresses directly (unified
 *               addressing); 16-byte aligned. The kernels move the data with
 *               16-byte loads and stores over the bus, with no separate copy.
 * src_dst       int32 [num_pairs][2], device or page-locked host memory.
 *               Precondition: the dst blocks are distinct and the source and
 *               destination regions do not overlap. A pair with src outside
 *               [0, src_blocks) or dst outside [0, dst_blocks) is skipped and
 *               reported in *err (PKV_DEV_BAD_PAIR).
 */
int kv_block_swap(void *dst_k, void *dst_v, const void *src_k, const void *src_v,
                  const int32_t *src_dst, int num_pairs, int num_kv_heads, int head_dim,
                  int block_size, int src_blocks, int dst_blocks, int dtype, int32_t *err,
                  void *stream);

/*
 * pkv_check_wait_timeout - diagnostic of the bounded waits. Every wait of the
 * decode kernels on an mbarrier gives up after about a second, stores
 * PKV_DEV_WAIT_TIMEOUT in *err and winds the kernel down instead of hanging.
 * This call runs that same wait on a barrier phase that nothing completes,
 * with a limit of limit_cycles SM clock cycles (1 .. 4e9), so the give-up path
 * can be exercised without any fault. err is a device pointer (not NULL); it
 * receives PKV_DEV_WAIT_TIMEOUT if it held 0. The kernel then returns and the
 * context stays usable. An fp16/bf16 decode called while *err holds
 * PKV_DEV_WAIT_TIMEOUT does no work (its output and the pools are left as they
 * were): the caller resets *err to 0 first. The fp32 path has no such waits.
 */
int pkv_check_wait_timeout(long long limit_cycles, int32_t *err, void *stream);

/* Static, human-readable text for a pkv_status value. */
const char *pkv_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* PKV_H_ */
