// Internal declarations shared by the library's translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace pkv {

// Everything a decode launch needs, as plain values (kernel parameter block).
struct DecodeArgs {
  void *out;
  const void *q;
  const void *k_pool;
  const void *v_pool;
  const int32_t *block_tables;
  const int32_t *context_lens;
  float *ws_o;    // [S][Hq][max_parts][D] partition outputs (normalised), or null
  float *ws_lse;  // [S][Hq][max_parts] partition log2-sum-exp, or null
  int num_seqs;
  int num_heads;
  int num_kv_heads;
  int head_dim;
  int block_size;
  int max_blocks;      // block-table row length
  int num_blocks;      // pool size in blocks
  int max_context_len; // host upper bound on context_lens
  int part_tokens;     // tokens per partition (multiple of 16)
  int max_parts;       // partitions of the longest allowed context
  float scale_log2;    // scale * log2(e): scores are kept in base-2 units
  int32_t *err;        // nullable device error word
  // Fused cache-append (or null): each sequence's newest token, [S][Hkv][D].
  // The decode writes it into the pool slot of token L-1 and attends over it.
  const void *k_new;
  const void *v_new;
  // Work list of the persistent decode kernel (written by the plan kernel):
  uint2 *work;         // [<= S*max_parts] {seq << 16 | partition, context length, or
                       //  1 << 31 | the leader's grp word for a group}
  int32_t *sched;      // [0] dispatch counter, [1] number of work-list entries,
                       // [2] first tail item, [3] pieces per tail item (< 2: none)
  // Partition merging (split contexts). Partitions are merged in chunks of
  // MERGE_CHUNK; a context with more than one chunk is merged in two levels.
  int32_t *merge_cnt;  // [S*Hkv][max_chunks] finished partitions per chunk; zeroed by the plan
  int32_t *merge_cnt2; // [S*Hkv] finished chunk merges; zeroed by the plan
  float *ws2_o;        // [S][Hq][max_chunks][D] chunk results (normalised), or null
  float *ws2_lse;      // [S][Hq][max_chunks] chunk log2-sum-exp, or null
  int max_chunks;      // ceil(max_parts / MERGE_CHUNK)
  int grid;            // CTAs of the decode grid (each takes item blockIdx.x first)
  // Shared-prefix groups (written by the plan kernel, read back by it):
  int max_group;       // most sequences one work item may attend together (1 = no groups)
  int32_t *grp;        // [S] 0: own entry; -1: member of an earlier leader's group;
                       //     > 0: leader, (members - 1) << 27 | shared 16-token tiles
  int32_t *grp_tiles;  // [S] a leader's group tiles: shared + every member's own
  int unit8;           // 1 when block_size % 16 == 8: a 16-token tile is two 8-token units
                       // that may sit in different blocks
  int wave_clusters;   // single-wave kernel: clusters per (sequence, KV head); above 1 each
                       // writes its merged partitions to a workspace slot (0 or 1: one)
  // Tail split of the persistent decode (see plan_kernel): the last items of
  // the work list are each attended as several pieces, merged when the last
  // piece of an item finishes.
  float *tail_o;       // [tail_slots][TAIL_COLS][D] piece outputs (normalised)
  float *tail_lse;     // [tail_slots][TAIL_COLS] piece log2-sum-exp
  int32_t *tail_cnt;   // [tail_slots] finished pieces per tail item; zeroed by the plan
  int tail_slots;      // pieces the tail region holds
};

constexpr int MERGE_CHUNK = 16;  // partitions merged together at the first level

// Tail split: a piece holds up to TAIL_COLS query-head rows (one work item's
// score columns); at most TAIL_MAX_PIECES pieces per call, TAIL_MAX_SPLIT per
// item, and each piece spans at least TAIL_MIN_PIECE_TILES 16-token tiles.
constexpr int TAIL_COLS = 8;
constexpr int TAIL_MAX_PIECES = 512;
constexpr int TAIL_MAX_SPLIT = 8;
constexpr int TAIL_MIN_PIECE_TILES = 8;

// Single-wave decode (decode_wave.cu): at most this many partitions per
// (sequence, KV head), one thread-block cluster of that many CTAs.
constexpr int WAVE_MAX_PARTS = 16;
// Contexts of at most this many 16-token tiles are attended one warp each.
constexpr int WAVE_WARP_TILES = 4;
// Under PKV_PARTITION_AUTO a single-wave partition holds at least this many
// tiles (one per warp).
constexpr int WAVE_MIN_PART_TILES = 4;
// Very long contexts: clusters of this many CTAs, several per (sequence, KV
// head), when that shortens each warp's chain of tiles by at least
// WAVE_SPLIT_MIN_GAIN tiles.
constexpr int WAVE_SPLIT_CLUSTER = 8;
constexpr int WAVE_SPLIT_MIN_GAIN = 16;
// Under the default selection, the single-wave kernel takes a call only if no
// warp gets more than this many 16-token tiles (its partitions are fixed per
// CTA; the persistent kernel balances ragged lengths instead).
constexpr int WAVE_MAX_WARP_CHAIN = 64;

// Decode workspace, in order: scheduling words (256 B), the work list, the
// per-sequence group words (two int32 per sequence), then (only when a
// context can span several partitions) the merge counters, the partition
// outputs with their log2-sum-exp values, and (only when a context can span
// several merge chunks) the chunk results, and last the tail-split region
// (piece counters, outputs and log2-sum-exp values of min(TAIL_MAX_PIECES,
// S * Hq * max_parts) pieces). Each region is 256-byte aligned.
struct WorkspaceLayout {
  size_t sched_off, work_off, grp_off, tcnt_off, to_off, tlse_off, cnt_off, cnt2_off, o_off,
      lse_off, o2_off, lse2_off, total;
  long long tail_slots;
};
WorkspaceLayout workspace_layout(long long S, long long Hq, long long D, long long max_parts);

// Plan + persistent decode (+ merge when split) for fp16 / bf16.
cudaError_t launch_wait_timeout_probe(long long limit_cycles, int32_t *err, cudaStream_t stream);
cudaError_t launch_decode_tc(const DecodeArgs &a, int dtype, const CUtensorMap &tmK,
                             const CUtensorMap &tmV, cudaStream_t stream);
cudaError_t launch_decode_simt_f32(const DecodeArgs &a, cudaStream_t stream);
// Single-wave decode for fp16 / bf16: `parts` partitions of a.part_tokens
// tokens per (sequence, KV head) on CTAs of `warps` (4 or 8) warps, or with
// warp_items one warp per (sequence, KV head) and one partition (4-warp
// CTAs). The workspace is not used.
cudaError_t launch_decode_wave(const DecodeArgs &a, int dtype, bool warp_items, int warps,
                               int parts, const CUtensorMap &tmK, const CUtensorMap &tmV,
                               cudaStream_t stream);
// How much of that work one wave holds: CTAs (warp_items, or parts == 1), or
// clusters of `parts` CTAs. 0 when the cluster shape cannot be resident.
cudaError_t decode_wave_capacity(const DecodeArgs &a, int dtype, bool warp_items, int warps,
                                 int parts, int *cap);
cudaError_t launch_merge(const DecodeArgs &a, int dtype, cudaStream_t stream);

cudaError_t launch_append(void *k_pool, void *v_pool, const void *k_new, const void *v_new,
                          const int64_t *slots, int num_tokens, int num_kv_heads, int row_bytes,
                          int block_size, int num_blocks, int32_t *err, cudaStream_t stream);
cudaError_t launch_block_swap(void *dst_k, void *dst_v, const void *src_k, const void *src_v,
                              const int32_t *pairs, int num_pairs, long long block_bytes,
                              int src_blocks, int dst_blocks, int32_t *err, cudaStream_t stream);
cudaError_t launch_block_copy(void *k_pool, void *v_pool, const int32_t *pairs, int num_pairs,
                              long long block_bytes, int num_blocks, int32_t *err,
                              cudaStream_t stream);

// Shared-memory bytes a decode_tc launch requests (for occupancy queries).
size_t decode_tc_smem_bytes(int head_dim);

}  // namespace pkv
