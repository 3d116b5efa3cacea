// Paged decode attention for fp16 / bf16 on sm_100a.
//
// Work is one (sequence, partition, KV head) item. The whole group of
// G = Hq/Hkv query heads that share the KV head is attended at once, so each
// K/V byte is read from HBM once per group.
//
// The block-by-block online softmax is the walk over the block table in page
// "PagedAttention Analysis" (ryotta.opik.net), section 3: look up each logical
// block's physical block, score it, update a running max / denominator /
// output. The partial last block is masked to the context length, which is
// the causal sum of page "PagedAttention" (newikis), section "Mathematical
// formulation".
//
// Scheduling
//   A one-CTA plan kernel turns context_lens into a compact work list of
//   (sequence, partition) pairs. Sequences of several partitions come first,
//   each with its short last partition first. Sequences of one partition
//   follow, largest first, with batch order kept within a size class. The plan
//   also resets the dispatch and merge counters. The decode kernel is
//   persistent, two CTAs per SM. Each CTA takes item blockIdx.x first, then
//   pulls items (pair x KV head) from an atomic counter until the list is
//   exhausted. Where the last items would leave most of the grid idle (a
//   remainder of at most half the grid, with one or two query heads per KV
//   head), the plan has each of them claimed as several pieces of consecutive
//   tiles, merged like partitions (plan_tail). Launches chain by programmatic
//   dependence: the plan is
//   launched while the previous call finishes (and waits for it before it
//   reads anything), and the decode grid's set-up overlaps the plan.
//
// Warp roles
//   Warp 4 is the scheduler. It resolves items ahead of use and posts them as
//   descriptors into a small ring: the work-list entry (with the context
//   length), the physical block ids of up to DESC_IDS tiles, and the group's q
//   rows, fetched by one bulk copy. In the last few items per CTA it holds at
//   most two descriptors, which spreads the final items over the CTAs. It
//   also keeps the partition count. When the consumers finish an item of a
//   split context, the scheduler publishes it (a device-scope fence and a
//   fetch-and-add on its chunk's counter). The scheduler warp that completes a
//   chunk of 16 partitions merges it right away, and the one that completes
//   the last chunk merges the chunks into `out`: the merges never queue behind
//   work items in a descriptor ring. The pieces of a tail-split item are
//   counted the same way, and the warp that completes the last piece merges
//   them. No CTA ever waits for another.
//   Warps 0-3 are consumers. Each owns a ring of stages in shared memory and
//   takes tiles w, w+4, w+8, ... of every item. Its lane 0 fills the ring
//   with TMA, completing on the stage's mbarrier:
//     - head_dim 128: one 3D copy per pool covers both 64-element halves of a
//       16-token tile;
//     - head_dim 64: one 2D copy per pool;
//     - block sizes that are odd multiples of 8: two 8-row boxes per
//       64-element half, one per 8-token unit, each from its own block.
//   The boxes are 128-byte swizzled. The fill runs ahead of the warp's math
//   across item boundaries. Every load lands in the issuing CTA only.
//
// Math (per tile, per consumer warp), fp32 accumulation:
//   S^T[16 tok][8] = K_tile[16][D] . Q^T[D][8]  mma.sync m16n8k16. K is the A
//     operand, read straight from the swizzled tile. The D axis is visited in
//     a lane-dependent order that Q's fragments follow too, which keeps every
//     shared load a conflict-free 16-byte access. Q (the group's heads,
//     zero-padded to 8) sits in registers for the whole item.
//   online softmax in base 2 on the accumulator fragment. The running max
//     moves only when a tile's max exceeds it by more than 2^8, which keeps
//     rescaling rare. Masked tokens get -inf, and their V rows are zeroed in
//     shared memory before they reach the tensor core.
//   O^T[D][8] += V^T[D][16] . P^T[16][8]  V^T via ldmatrix.trans; P^T from the
//     score fragment via movmatrix.trans. For bf16, P is split into hi + lo
//     bf16 parts (two MMAs), so the weights keep ~16 significant bits; fp16
//     keeps one operand (11 bits).
// At the end of an item the consumer warps' (max, sum, output) are combined in
// shared memory. The result goes to `out` when the sequence has one
// partition, and otherwise to the workspace as (normalised o_p,
// log2-sum-exp). The consumers meet at three barriers per item: a vote at
// its start (which also orders the reuse of the combine area), one after
// their partial rows are stored and one after the per-warp weights are.
// Every wait is bounded: one that gives up sets an error status and a
// CTA-wide stop flag, and the kernel winds down, first waiting (bounded) for
// the copies it still has in flight.
#include <climits>
#include <type_traits>

#include "pkv_device.cuh"
#include "pkv_internal.h"

namespace pkv {
namespace {

constexpr int TILE = 16;                 // tokens per tile (mma M for QK, K for PV)
constexpr int NCW = 4;                   // consumer warps
constexpr int THREADS = (NCW + 1) * 32;  // + one scheduler warp
constexpr int NSLOT = 3;                 // item descriptors in flight
// Near the end of the work list a CTA holds at most two work descriptors (the
// one being consumed and the next), so that the last items are spread over
// the CTAs instead of queued in a few of them. "Near" = fewer than this many
// items per CTA left.
constexpr int END_ITEMS_PER_CTA = 6;
// Block ids a descriptor carries: one per 16-token tile, or one per 8-token
// unit when the block size is an odd multiple of 8 (128 tiles cover a
// 2048-token partition). Further ids are read from the table when their tile
// is fetched.
constexpr int DESC_IDS = 128;
constexpr int IDS_PER_LANE = DESC_IDS / 32;
static_assert(DESC_IDS % 32 == 0, "ids are fetched 32 at a time");
constexpr int BOX_COLS = 64;             // elements per TMA box row (128 bytes)
constexpr int HALF_BYTES = TILE * 128;   // one box: 16 rows x 128 bytes
constexpr int PLAN_THREADS = 256;
constexpr float RESCALE_SLACK = 8.f;     // lazy max: rescale only past 2^8 growth

// Descriptor kinds (in ItemDesc::kind).
constexpr int KIND_WORK = 0;         // attend one (sequence, partition, KV head)
constexpr int KIND_NOP = 1;          // keeps the ring turning while the last items finish
constexpr int KIND_END = 2;          // no more descriptors
constexpr int PLAN_BUCKETS = 64;     // size classes for ordering the short last partitions

// Most sequences one work item attends together (a shared-prefix group).
constexpr int MAX_MEMBERS = 8;

// One entry of the scheduler -> consumer descriptor ring. A work item attends
// `members` sequences s, s+1, ... (one, or a group that shares its first `sh`
// tiles) for one KV head. Its tiles are numbered group-wide: the shared tiles
// 0 .. sh-1 (tokens 0 .. 16*sh-1 of every member), then member m's own tiles
// own[m] .. own[m+1]-1 (its tokens from 16*sh on). Partition p covers group
// tiles tile0 .. tile0 + n_tiles - 1.
struct alignas(16) ItemDesc {
  int kind, s, p, h, n_tiles, nparts;
  int members;   // sequences attended by this item
  int tile0;     // group tile of the partition's first tile
  int sh;        // shared tiles (0 for one sequence)
  int own[MAX_MEMBERS + 1];  // first own tile of each member; own[members] = all tiles
  int len[MAX_MEMBERS];      // members' context lengths
  int ids[DESC_IDS];  // physical block of tile (or 8-token unit) t; -1 past the context
  int tail;  // piece slot of a tail-split item (p = piece, nparts = pieces), or -1
};

// Shared-memory plan of one CTA (offsets from the 1024-aligned base). NH is
// the number of score columns (query-head rows) an item carries: the G heads
// of one sequence (NH = 4 serves G = 3, 4), or with NH = 8 the heads of up to
// 8 / G sequences that share a prefix (G = 1, 2; one sequence for G = 5..8).
template <int D, int NH>
struct TcShape {
  static constexpr int HALVES = D / BOX_COLS;
  static constexpr int KT_BYTES = HALVES * HALF_BYTES;   // one K (or V) tile
  static constexpr int STAGE_BYTES = 2 * KT_BYTES;       // K + V
  static constexpr int ACC_STRIDE = D + 4;               // padded combine row (floats)
  static constexpr int CW_FLOATS = NH * ACC_STRIDE + 2 * NH;  // acc[NH][D+4], m[NH], l[NH]
  // With 8 columns a warp's partial result of an item is combined from the
  // ring stage of its last tile, which it refills only after the next item's
  // vote: a combine area of its own (4 x 8 x 132 floats) would leave room for
  // two stages only. With 4 columns the area fits beside three stages, and a
  // warp refills its last stage at once.
  static constexpr bool RING_COMBINE = NH >= 8;
  // Shared-prefix groups (several sequences per item) only with 8 columns.
  static constexpr bool GROUPS = NH >= 8;
  static_assert(!RING_COMBINE || CW_FLOATS * 4 <= STAGE_BYTES, "a stage holds the rows");
  // With 8 columns, items of at most SMALL_COLS columns (one sequence with
  // G <= 2) still combine in a small area of their own and hold no stage.
  static constexpr int SMALL_COLS = 2;
  static constexpr int SMALL_CW = SMALL_COLS * ACC_STRIDE + 2 * SMALL_COLS;
  static constexpr int COMBINE_BYTES = NCW * (RING_COMBINE ? SMALL_CW : CW_FLOATS) * 4;
  // weights [NH][NCW], log2-sum-exp [NH], each warp's combine stage [NCW]
  static constexpr int SCALES_BYTES = (NH * (NCW + 1) + NCW) * 4;
  // An item of one sequence gets its newest K and V rows (fused append)
  // with its q rows; a group's members read theirs from k_new / v_new.
  static constexpr int QROWS_BYTES = NH * D * 2;  // the q rows of every member
  static constexpr int QBUF_BYTES = QROWS_BYTES + 2 * D * 2;
  static constexpr int FIXED = COMBINE_BYTES + ((SCALES_BYTES + 15) & ~15) +
                               NSLOT * QBUF_BYTES + NSLOT * (int)sizeof(ItemDesc) + 64 * 8 +
                               1024 + 64;
  // As many stages as fit two CTAs per SM, at most 6. An SM has 228 KB of
  // shared memory and each CTA also reserves 1 KB, so a CTA may use ~113 KB.
  static constexpr int CTA_SMEM_BUDGET = 228 * 1024 / 2 - 1024 - 256;
  static constexpr int NSTAGE_FIT = (CTA_SMEM_BUDGET - FIXED) / (NCW * STAGE_BYTES);
  static constexpr int NSTAGE = NSTAGE_FIT > 6 ? 6 : NSTAGE_FIT;
  static_assert(NSTAGE >= 3, "ring too shallow");
  static constexpr int RING_BYTES = NCW * NSTAGE * STAGE_BYTES;
  static constexpr int COMBINE_OFF = RING_BYTES;
  static constexpr int SCALES_OFF = COMBINE_OFF + COMBINE_BYTES;
  static constexpr int QBUF_OFF = SCALES_OFF + ((SCALES_BYTES + 15) & ~15);
  static constexpr int DESC_OFF = QBUF_OFF + NSLOT * QBUF_BYTES;
  static constexpr int BAR_OFF = DESC_OFF + NSLOT * (int)sizeof(ItemDesc);
  static constexpr int NBARS = NCW * NSTAGE + 2 * NSLOT;
  static_assert(NBARS <= 64, "barrier area");
  static constexpr int SMEM_BYTES = BAR_OFF + NBARS * 8 + 1024;  // + alignment slack
  static_assert(SMEM_BYTES <= CTA_SMEM_BUDGET, "two CTAs per SM");
  static_assert(NH <= TAIL_COLS, "a tail piece slot holds every column of an item");
  static_assert(QBUF_OFF % 16 == 0 && DESC_OFF % 16 == 0 && BAR_OFF % 8 == 0, "alignment");
};

__device__ __forceinline__ uint32_t pack_pair(int s, int p) {
  return (static_cast<uint32_t>(s) << 16) | static_cast<uint32_t>(p);
}

// Tiles per partition of an entry. One sequence uses the call's partition
// length. A group of sequences that share a prefix (see plan_group_round) spans its
// shared tiles once plus every member's own tiles; it uses partitions long
// enough that their number never exceeds max_parts, so each member's partial
// results fit its workspace rows.
__device__ __forceinline__ int group_part_tiles(const DecodeArgs &a, bool grouped, int tiles) {
  const int pt = a.part_tokens / TILE;
  return grouped ? max(pt, (tiles + a.max_parts - 1) / a.max_parts) : pt;
}

// Inclusive prefix maximum over the plan block (one value per thread).
__device__ __forceinline__ int plan_block_max_scan(int v, int *wmax) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int y = __shfl_up_sync(FULL_MASK, v, off);
    if (lane >= off) v = max(v, y);
  }
  if (lane == 31) wmax[warp] = v;
  __syncthreads();
  int before = INT_MIN;
  for (int w = 0; w < warp; ++w) before = max(before, wmax[w]);
  __syncthreads();  // wmax is reused by the next scan
  return max(v, before);
}

// Shared-prefix groups, found by the plan kernel when a.max_group > 1.
//
// Sequences that share blocks (the samples of one prompt, the beams of one
// request, requests that hit the same cached prefix: page "PagedAttention
// Analysis", section 4, and the copy-on-write section of page "추론 엔진에서의
// 메모리 가상화") point to the same physical blocks from the start of their
// block tables. A physical block holds one set of K/V values whoever reads it,
// so adjacent sequences whose table entries agree up to some block can be
// attended by one work item that reads those shared tiles once, with every
// member's query rows side by side in the tensor-core N dimension.
//
// For each round of PLAN_THREADS sequences:
//  - psh(s): the tiles of 16 tokens that sequence s shares with s-1: the
//    tokens of all blocks before the first table entry where they differ,
//    capped at both lengths and rounded down to whole tiles. With a fused
//    append each sequence's newest token is excluded (it is written in this
//    call, so it is never read as shared).
//  - A run is a maximal stretch of sequences each sharing at least one tile
//    with its predecessor; runs do not cross rounds. A run is cut into groups
//    of at most a.max_group members, and a group's shared length is the
//    smallest psh inside it.
//  - a.grp[s] = 0 for a sequence on its own, (members - 1) << 27 | shared
//    tiles for a group's first member (its leader), -1 for the other members;
//    a.grp_tiles[leader] = shared tiles + every member's own tiles.
// The table comparison touches only candidate pairs (equal first entries) and
// only the entries that both sequences' shared span covers, spread over all
// threads of the block.
// One round of PLAN_THREADS sequences (thread tid holds sequence s = r0 + tid,
// of clamped length L) that has at least one candidate pair (cand: s-1 and s
// may share `cap` tiles and their first table entries agree). Sets this
// thread's group word and, for a leader, the group's tiles, and stores both
// in a.grp / a.grp_tiles for the plan's second pass.
template <typename BlockScan>
__device__ __noinline__ void plan_group_round(const DecodeArgs &a, int s, int L, int cap,
                                              bool cand, BlockScan block_scan, int &word,
                                              int &gtiles) {
  __shared__ int c_seq[PLAN_THREADS];     // candidate pairs (s-1, s): s
  __shared__ int c_mis[PLAN_THREADS];     // first differing block (or the blocks compared)
  __shared__ int g_cnt[PLAN_THREADS];     // members of the group a thread leads
  __shared__ int g_sh[PLAN_THREADS];      // its shared tiles
  __shared__ int g_own[PLAN_THREADS];     // its members' own tiles
  __shared__ int wmax[PLAN_THREADS / 32];
  const int tid = threadIdx.x;
  const int S = a.num_seqs, B = a.block_size;
  const int nblk = cand ? (cap * TILE + B - 1) / B : 0;  // blocks covering the span
  int ncand;
  const int ci = block_scan(cand ? 1 : 0, ncand);  // this candidate's index
  if (cand) {
    c_seq[ci] = s;
    c_mis[ci] = nblk;
  }
  g_cnt[tid] = 0;
  g_sh[tid] = INT_MAX;
  g_own[tid] = 0;
  __syncthreads();
  // Every comparison of every candidate. Warp w takes candidates w, w + 8,
  // ... in batches of CMP_CANDS; lane l compares blocks 1 + l, 33 + l, ... of
  // each, CMP_CHUNKS chunks of 32 blocks at a time, with all of a batch's
  // loads issued before the comparisons. A warp minimum gives the first
  // differing block.
  constexpr int NWARP = PLAN_THREADS / 32, CMP_CANDS = 16, CMP_CHUNKS = 2;
  const int lane = tid & 31, warp = tid >> 5;
  for (int c0 = warp; c0 < ncand; c0 += NWARP * CMP_CANDS) {
    const int32_t *rows[CMP_CANDS];
    int nb[CMP_CANDS], mis[CMP_CANDS];
#pragma unroll
    for (int k = 0; k < CMP_CANDS; ++k) {
      const int c = c0 + k * NWARP;
      rows[k] = a.block_tables + (size_t)(c < ncand ? c_seq[c] : 1) * a.max_blocks;
      nb[k] = c < ncand ? c_mis[c] : 0;  // blocks covering the candidate's span
      mis[k] = nb[k];
    }
    int longest = 0;
#pragma unroll
    for (int k = 0; k < CMP_CANDS; ++k) longest = max(longest, nb[k]);
    for (int j0 = 1; j0 < longest; j0 += 32 * CMP_CHUNKS) {
      int va[CMP_CANDS][CMP_CHUNKS], vb[CMP_CANDS][CMP_CHUNKS];
#pragma unroll
      for (int k = 0; k < CMP_CANDS; ++k)
#pragma unroll
        for (int q = 0; q < CMP_CHUNKS; ++q) {
          const int j = j0 + lane + 32 * q;
          const bool in = j < nb[k] && j < mis[k];
          va[k][q] = in ? rows[k][j] : 0;
          vb[k][q] = in ? (rows[k] - a.max_blocks)[j] : 0;  // row s-1 precedes row s
        }
#pragma unroll
      for (int k = 0; k < CMP_CANDS; ++k) {
        int first = mis[k];
#pragma unroll
        for (int q = 0; q < CMP_CHUNKS; ++q) {
          const int j = j0 + lane + 32 * q;
          if (j < nb[k] && va[k][q] != vb[k][q]) first = min(first, j);
        }
        mis[k] = __reduce_min_sync(FULL_MASK, first);
      }
    }
#pragma unroll
    for (int k = 0; k < CMP_CANDS; ++k) {
      const int c = c0 + k * NWARP;
      if (lane == 0 && c < ncand) c_mis[c] = mis[k];
    }
  }
  __syncthreads();
  const int psh = cand ? min(c_mis[ci] * B / TILE, cap) : 0;
  const bool linked = psh > 0;  // never for tid 0: runs do not cross rounds
  const int run = plan_block_max_scan(linked ? -1 : tid, wmax);
  const int lead = run + (tid - run) / a.max_group * a.max_group;
  if (s < S) {
    atomicAdd(&g_cnt[lead], 1);
    if (tid != lead) atomicMin(&g_sh[lead], psh);
  }
  __syncthreads();
  const int members = g_cnt[lead];
  const int sh = members > 1 ? g_sh[lead] : 0;
  if (s < S && members > 1) atomicAdd(&g_own[lead], (L - sh * TILE + TILE - 1) / TILE);
  __syncthreads();
  word = 0;
  gtiles = 0;
  if (s < S) {
    if (members > 1) word = tid == lead ? ((members - 1) << 27) | sh : -1;
    if (word > 0) gtiles = sh + g_own[lead];
    a.grp[s] = word;
    if (word > 0) a.grp_tiles[s] = gtiles;
  }
  __syncthreads();  // the shared arrays are rewritten by the next round
}

// The work list of a batch of at most 32 sequences with no shared-prefix
// groups, built by one warp with shuffles instead of block barriers: the same
// list plan_kernel builds (lane s holds sequence s).
__device__ __noinline__ void plan_small(const DecodeArgs &a, int lane) {
  const int S = a.num_seqs;
  const int s = lane;
  int raw = 0, L = 0;
  if (s < S) {
    raw = a.context_lens[s];
    L = effective_len(raw, a.max_context_len, a.max_blocks, a.block_size, nullptr);
  }
  const bool bad_len = __any_sync(FULL_MASK, s < S && L < raw);
  const int pt = max(1, a.part_tokens / TILE);  // tiles per partition
  const int tiles = (L + TILE - 1) / TILE;
  const int np = s < S ? max(1, (tiles + pt - 1) / pt) : 0;
  // region 1: sequences of several partitions, in batch order, each with its
  // short last partition first
  const int nm = np > 1 ? np : 0;
  int incl = nm;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int y = __shfl_up_sync(FULL_MASK, incl, off);
    if (lane >= off) incl += y;
  }
  const int total_m = __shfl_sync(FULL_MASK, incl, 31);
  uint2 *const list = a.work;
  if (nm > 0) {
    const int o = incl - nm;
    list[o] = make_uint2(pack_pair(s, np - 1), (uint32_t)L);
    for (int q = 0; q < np - 1; ++q) list[o + 1 + q] = make_uint2(pack_pair(s, q), (uint32_t)L);
  }
  // region 2: one-partition sequences, larger size class first, batch order
  // within a class (a sequence of length 0 is one empty entry)
  const int bkt = np == 1 ? (PLAN_BUCKETS - 1) -
                                min(PLAN_BUCKETS - 1, tiles * (PLAN_BUCKETS - 1) / pt)
                          : INT_MAX;
  int rank = 0;
  for (int j = 0; j < 32; ++j) {
    const int b = __shfl_sync(FULL_MASK, bkt, j);
    if (b < bkt || (b == bkt && j < lane)) ++rank;
  }
  if (np == 1) list[total_m + rank] = make_uint2(pack_pair(s, 0), (uint32_t)L);
  const int total = total_m + __popc(__ballot_sync(FULL_MASK, np == 1));
  if (a.merge_cnt) {
    const int n1 = S * a.num_kv_heads * a.max_chunks;
    for (int i = lane; i < n1; i += 32) a.merge_cnt[i] = 0;
    for (int i = lane; i < S * a.num_kv_heads; i += 32) a.merge_cnt2[i] = 0;
  }
  if (lane == 0) {
    a.sched[0] = a.grid;  // items 0 .. grid-1 are each CTA's first, taken without the counter
    a.sched[1] = total;
    if (bad_len) report(a.err, PKV_DEV_CONTEXT_LEN);
  }
}

// Tail split, decided by every thread of the plan block alike once the work
// list (total entries, the first total_m of several partitions) is written.
// The CTAs take items in list order, so the last wave holds the r = items mod
// grid last items (the smallest, by the size classes) while the other CTAs
// run out of work. When r is at most half the grid and those items are long,
// each of them is attended as k = min(grid / r, ...) pieces of consecutive
// tiles instead, so the last wave spreads over about r * k CTAs; the pieces'
// partial results (in the tail region) are merged when an item's last piece
// finishes. Only one-partition entries are split, and every piece keeps at
// least TAIL_MIN_PIECE_TILES tiles (the last entry is the smallest). The plan
// asks for it only where groups may form (8 score columns, one or two query
// heads per KV head): there an item may carry a whole group of sequences and
// items are few and long. (With 4 columns the pieces' fixed costs outweighed
// the gain: a beam-search step took 4 % longer.) Zeroes the counters of the
// items it splits.
__device__ __noinline__ void plan_tail(const DecodeArgs &a, int total, int total_m,
                                       int &tail_first, int &tail_split) {
  const long long items_ll = (long long)total * a.num_kv_heads;
  if (a.tail_cnt == nullptr || items_ll <= a.grid || items_ll >= INT_MAX) return;
  const int items = static_cast<int>(items_ll);
  const int r = items % a.grid;
  if (r == 0) return;
  int k = min(TAIL_MAX_SPLIT, min(a.grid / r, a.tail_slots / r));
  const int first = items - r;
  if (k < 2 || first < total_m * a.num_kv_heads) return;
  const uint2 last = a.work[total - 1];  // (written before the plan's last barrier)
  const int ls = min(static_cast<int>(last.x >> 16), a.num_seqs - 1);
  const int tiles =
      (last.y >> 31) != 0 ? a.grp_tiles[ls] : (static_cast<int>(last.y) + TILE - 1) / TILE;
  k = min(k, tiles / TAIL_MIN_PIECE_TILES);
  if (k < 2) return;
  tail_first = first;
  tail_split = k;
  for (int i = threadIdx.x; i < r; i += blockDim.x) a.tail_cnt[i] = 0;
}

// Build the work list in two regions.
//  1. Entries of several partitions: all their partitions, entry by entry,
//     the short last partition first. Their merges then complete while the
//     list is still being worked through.
//  2. Entries of one partition, ordered by size, largest first (a counting
//     sort over PLAN_BUCKETS size classes). They need no merge, and handing out
//     the largest first and the smallest last keeps the CTAs' finishing times
//     close. The sort is stable: within a size class the entries keep batch
//     order. A sequence of length 0 is one (empty) entry, so that its output
//     is still written.
// An entry is one sequence, or, when a.max_group > 1, one group of adjacent
// sequences that share their first blocks (plan_group_round): the group's leader
// carries it and the other members have no entry. Each entry carries the
// sequence's clamped length, or the leader's group word. Sequences are taken
// in rounds of PLAN_THREADS (thread t holds sequence round*PLAN_THREADS + t),
// so that thread order is sequence order. The merge counters are reset here
// too, and the tail split is decided (plan_tail).
//
// This grid is the programmatic dependent of what precedes it, typically the
// previous decode call, and may start while that call is still running. It
// waits for that grid to complete (griddepcontrol.wait) before it reads or
// writes global memory: the context lengths may come from the kernel before
// it, and the workspace may still be in use by the previous call.
// TAIL: the decode kernel it feeds has the 8-column layout, which reads the
// tail-split words (written whenever the block plans, i.e. always when groups
// may form).
template <bool TAIL>
__global__ void __launch_bounds__(PLAN_THREADS) plan_kernel(const DecodeArgs a) {
  constexpr int NW = PLAN_THREADS / 32;
  __shared__ int wsum[NW];
  __shared__ int hist[PLAN_BUCKETS];        // count, then running start of each size class
  __shared__ int wcnt[NW][PLAN_BUCKETS];    // per-warp counts of a round, then their offsets
  __shared__ int total_m_s;
  __shared__ int total_s;
  __shared__ int bad_len;  // a context length was clamped: reported after the wait
  pdl_launch_dependents();  // the decode grid may launch; it waits for this grid to finish
  pdl_wait();
  uint2 *const list = a.work;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int S = a.num_seqs;
  const bool grouping = a.max_group > 1;
  if (!grouping && S <= 32) {  // a small batch: warp 0 plans alone (no block barriers)
    if (warp == 0) plan_small(a, lane);
    return;
  }
  if (tid < PLAN_BUCKETS) hist[tid] = 0;
  if (tid == 0) bad_len = 0;
  __syncthreads();
  const int max_tiles = max(1, a.part_tokens / TILE);
  // size class of a one-partition entry of `tiles` tiles: bigger -> smaller class
  auto bucket = [&](int tiles) {
    return (PLAN_BUCKETS - 1) - min(PLAN_BUCKETS - 1, tiles * (PLAN_BUCKETS - 1) / max_tiles);
  };
  // Exclusive block-wide prefix sum of v; `total` receives the sum.
  auto block_scan = [&](int v, int &total) {
    int f = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(FULL_MASK, f, off);
      if (lane >= off) f += y;
    }
    if (lane == 31) wsum[warp] = f;
    __syncthreads();
    if (warp == 0) {
      int w = lane < NW ? wsum[lane] : 0;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(FULL_MASK, w, off);
        if (lane >= off) w += y;
      }
      if (lane < NW) wsum[lane] = w;  // inclusive prefix over warps
    }
    __syncthreads();
    const int excl = (warp ? wsum[warp - 1] : 0) + f - v;
    total = wsum[NW - 1];
    __syncthreads();  // wsum is reused by the next scan
    return excl;
  };
  auto eff_len = [&](int s) {
    return effective_len(a.context_lens[s], a.max_context_len, a.max_blocks, a.block_size,
                         nullptr);
  };

  // Tiles and partitions of sequence s's entry from its group word g (np = 0:
  // no entry, a group member other than the leader). `word` is the entry's
  // second field.
  auto entry_shape = [&](int L, int g, int gtiles, int &np, int &tiles, uint32_t &word) {
    word = (uint32_t)L;
    tiles = (L + TILE - 1) / TILE;
    if (g < 0) {
      np = 0;
      return;
    }
    if (g > 0) {
      tiles = gtiles;
      word = 0x80000000u | (uint32_t)g;
    }
    const int ptg = group_part_tiles(a, g > 0, tiles);
    np = max(1, (tiles + ptg - 1) / ptg);  // an empty sequence still has its (empty) entry
  };

  // pass 1: the shared-prefix groups of each round, the region-1 entry count
  // and the size-class histogram of region 2. With groups possible, each
  // thread loads its predecessor's length and both first table entries with
  // its own length; a round where no pair of first entries agrees costs one
  // more barrier.
  const int newest = a.k_new != nullptr ? 1 : 0;
  bool any_group = false;  // (uniform) a group formed: the words are in a.grp
  int nm = 0;
  int L1 = 0, word1 = 0, gtiles1 = 0;  // this thread's last pass-1 values
  for (int r0 = 0; r0 < S; r0 += PLAN_THREADS) {
    const int s = r0 + tid;
    int raw = 0, raw_prev = 0;
    int32_t b_this = 0, b_prev = 0;
    if (s < S) {
      raw = a.context_lens[s];
      if (grouping && tid > 0) {  // (runs do not cross rounds)
        const int32_t *bt = a.block_tables + (size_t)s * a.max_blocks;
        raw_prev = a.context_lens[s - 1];
        b_this = bt[0];
        b_prev = (bt - a.max_blocks)[0];  // row s-1 precedes row s
      }
    }
    const int L = s < S ? effective_len(raw, a.max_context_len, a.max_blocks, a.block_size,
                                        nullptr)
                        : 0;
    if (s < S && L < raw) bad_len = 1;
    int word = 0, gtiles = 0;
    if (grouping) {
      int cap = 0;  // tiles the pair (s-1, s) could share
      if (s < S && tid > 0)
        cap = (min(L, effective_len(raw_prev, a.max_context_len, a.max_blocks, a.block_size,
                                    nullptr)) -
               newest) / TILE;
      const bool cand = cap > 0 && b_this == b_prev;
      if (__syncthreads_or(cand)) {
        if (!any_group) {  // the earlier rounds had no group: record them as single sequences
          for (int i = tid; i < r0; i += PLAN_THREADS) a.grp[i] = 0;
          any_group = true;
        }
        plan_group_round(a, s, L, cap, cand, block_scan, word, gtiles);
      } else if (any_group && s < S) {
        a.grp[s] = 0;
      }
    }
    L1 = L;
    word1 = word;
    gtiles1 = gtiles;
    if (s < S) {
      int np, tiles;
      uint32_t w;
      entry_shape(L, word, gtiles, np, tiles, w);
      if (np > 1)
        nm += np;
      else if (np == 1)
        atomicAdd(&hist[bucket(tiles)], 1);
    }
  }
  int total_m;
  block_scan(nm, total_m);
  // running start of each size class (exclusive scan of hist, after region 1)
  if (warp == 0) {
    const int h0 = hist[2 * lane], h1 = hist[2 * lane + 1];
    int v = h0 + h1;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(FULL_MASK, v, off);
      if (lane >= off) v += y;
    }
    const int excl = v - h0 - h1;
    hist[2 * lane] = total_m + excl;
    hist[2 * lane + 1] = total_m + excl + h0;
    if (lane == 31) total_s = total_m + v;
  }
  if (tid == 0) total_m_s = 0;
  __syncthreads();

  // pass 2: write the entries, one round of PLAN_THREADS sequences at a time
  for (int r0 = 0; r0 < S; r0 += PLAN_THREADS) {
    const int s = r0 + tid;
    int np = 0, bkt = -1;
    uint32_t word = 0;
    if (s < S) {
      int n, tiles;
      // (one round: this thread's word from pass 1 is still in registers)
      const int g = !any_group ? 0 : S <= PLAN_THREADS ? word1 : a.grp[s];
      const int gt = g <= 0 ? 0 : S <= PLAN_THREADS ? gtiles1 : a.grp_tiles[s];
      entry_shape(S <= PLAN_THREADS ? L1 : eff_len(s), g, gt, n, tiles, word);
      if (n > 1)
        np = n;
      else if (n == 1)
        bkt = bucket(tiles);
    }
    // region 1: this round's entries after the previous rounds'
    int round_m;
    const int om = total_m_s + block_scan(np, round_m);
    if (np > 0) {
      list[om] = make_uint2(pack_pair(s, np - 1), word);
      for (int q = 0; q < np - 1; ++q) list[om + 1 + q] = make_uint2(pack_pair(s, q), word);
    }
    // region 2: rank among this warp's lanes of the same class, then the
    // earlier warps' counts, then the class's running start
    for (int i = tid; i < NW * PLAN_BUCKETS; i += PLAN_THREADS) (&wcnt[0][0])[i] = 0;
    __syncthreads();
    const unsigned same = __match_any_sync(FULL_MASK, bkt);
    const int rank = __popc(same & ((1u << lane) - 1u));
    if (bkt >= 0 && lane == 31 - __clz(same)) wcnt[warp][bkt] = __popc(same);
    __syncthreads();
    if (tid < PLAN_BUCKETS) {
      int start = hist[tid];
      for (int w = 0; w < NW; ++w) {
        const int c = wcnt[w][tid];
        wcnt[w][tid] = start;
        start += c;
      }
      hist[tid] = start;
    }
    if (tid == 0) total_m_s += round_m;
    __syncthreads();
    if (bkt >= 0) list[wcnt[warp][bkt] + rank] = make_uint2(pack_pair(s, 0), word);
    __syncthreads();  // wcnt and total_m_s are rewritten by the next round
  }
  const int total = total_s;
  int tail_first = 0, tail_split = 0;
  if (TAIL && grouping) plan_tail(a, total, total_m, tail_first, tail_split);
  if (a.merge_cnt) {
    const int n1 = S * a.num_kv_heads * a.max_chunks;
    for (int i = tid; i < n1; i += PLAN_THREADS) a.merge_cnt[i] = 0;
    for (int i = tid; i < S * a.num_kv_heads; i += PLAN_THREADS) a.merge_cnt2[i] = 0;
  }
  if (tid == 0) {
    a.sched[0] = a.grid;  // items 0 .. grid-1 are each CTA's first, taken without the counter
    a.sched[1] = total;
    if (TAIL) {
      a.sched[2] = tail_first;
      a.sched[3] = tail_split;
    }
    if (bad_len) report(a.err, PKV_DEV_CONTEXT_LEN);
  }
}

// Wait for an mbarrier phase, or give up. A wait gives up when the CTA-wide
// abort flag is set, or when it has spun for WAIT_LIMIT_CYCLES; in the second
// case it sets the flag and reports PKV_DEV_WAIT_TIMEOUT. Either way the
// caller leaves its loop, so a failure ends the kernel instead of stalling.
__device__ __forceinline__ bool wait_or_abort(uint32_t bar, uint32_t parity,
                                              volatile int *abort_flag, int32_t *err,
                                              long long limit = WAIT_LIMIT_CYCLES) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (*abort_flag) return false;
    if (clock64() - t0 > limit) {
      *abort_flag = 1;
      report(err, PKV_DEV_WAIT_TIMEOUT);
      return false;
    }
  }
  return true;
}

// Bounded wait with no abort check, for the copies still in flight when a
// warp stops after a wait gave up: it returns once the phase completes or
// after DRAIN_LIMIT_CYCLES, whichever is first.
constexpr long long DRAIN_LIMIT_CYCLES = 20000000LL;
__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity))
    if (clock64() - t0 > DRAIN_LIMIT_CYCLES) return false;
  return true;
}

// Diagnostic: one block waits, through wait_or_abort, on an mbarrier phase
// that nothing completes, with a short limit. The wait must give up, set the
// abort flag and report PKV_DEV_WAIT_TIMEOUT, and the kernel must return; the
// decode kernels' waits run the same code with the long limit.
__global__ void wait_timeout_probe_kernel(long long limit, int32_t *err) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  const uint32_t b = smem_addr(&bar);
  if (threadIdx.x == 0) {
    mbar_init(b, 1);  // one arrival expected; none ever comes
    fence_mbar_init();
    abort_flag = 0;
  }
  __syncthreads();
  const bool ok = wait_or_abort(b, 0, &abort_flag, err, limit);
  if (ok && threadIdx.x == 0) report(err, PKV_DEV_BAD_PAIR);  // a phase completed: wrong
}

// Non-blocking test of an mbarrier phase.
__device__ __forceinline__ bool mbar_test(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n"
      "  .reg .pred p;\n"
      "  mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      "  selp.u32 %0, 1, 0, p;\n"
      "}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// Add `bytes` to the current phase's expected transaction count, without an
// arrival (the phase completes after the arrivals and all the bytes).
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

// Bulk copy global -> shared (no tensor map), completing on an mbarrier.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void *src, uint32_t bytes,
                                          uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          dst),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
      : "memory");
}

// Barrier among the consumer warps only (the scheduler warp keeps running).
__device__ __forceinline__ void consumers_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(NCW * 32) : "memory");
}

// Consumer barrier that also returns the AND of `v` over all consumer threads,
// so that every consumer warp takes the same exit decision.
__device__ __forceinline__ bool consumers_all(bool v) {
  uint32_t r;
  asm volatile(
      "{\n"
      "  .reg .pred pin, pout;\n"
      "  setp.ne.u32 pin, %1, 0;\n"
      "  bar.red.and.pred pout, 1, %2, pin;\n"
      "  selp.u32 %0, 1, 0, pout;\n"
      "}\n"
      : "=r"(r)
      : "r"((uint32_t)v), "n"(NCW * 32)
      : "memory");
  return r != 0;
}

// Merge entries [q0, q1) (at most MERGE_CHUNK) of one work item's KV head,
// for the G query heads of each of its `members` sequences s, s+1, ...:
// o = sum_q 2^(lse_q - lse) o_q with lse = log2 sum_q 2^lse_q. The sources
// were written by other CTAs; they are read from L2 (ld.global.cg). The
// result goes to `out` (final), or to chunk entry `dst_idx` of the
// second-level arrays as (o, lse). Threads tid = 0 .. nthreads-1 share it.
// BY_PIECE: the entries are pieces q0 .. q1-1 of a tail-split item in the
// tail region (src_stride unused).
template <typename T, int D, bool BY_PIECE = false>
__device__ __noinline__ void merge_range(const DecodeArgs &a, int s, int h, int G, int members,
                                         const float *src_o, const float *src_lse,
                                         int src_stride, int q0, int q1, bool final_out,
                                         int dst_idx, int tid, int nthreads) {
  constexpr int V = D / 4;  // float4 columns per head row
  T *const out = static_cast<T *>(a.out);
  const int n_q = q1 - q0;
  for (int idx = tid; idx < members * G * V; idx += nthreads) {
    const int n = idx / V;
    const int cv = idx - n * V;
    const int mem = n / G;
    const size_t row = (size_t)(s + mem) * a.num_heads + h * G + (n - mem * G);
    // Entry q of this row: a sequence row's partitions are consecutive
    // (src_stride per row); a tail item's pieces hold TAIL_COLS rows each, the
    // item's column n in row n of each piece.
    const size_t base = BY_PIECE ? (size_t)q0 * TAIL_COLS + n : row * src_stride + q0;
    constexpr size_t qs = BY_PIECE ? TAIL_COLS : 1;
    const float *lse = src_lse + base;
    const float4 *po = reinterpret_cast<const float4 *>(src_o + base * D) + cv;
    // All of the entries' loads are issued before the first is used.
    float lq[MERGE_CHUNK];
    float4 vq[MERGE_CHUNK];
#pragma unroll
    for (int q = 0; q < MERGE_CHUNK; ++q) {
      lq[q] = q < n_q ? __ldcg(lse + q * qs) : -INFINITY;
      vq[q] = q < n_q ? __ldcg(po + q * qs * V) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    float M = -INFINITY;
#pragma unroll
    for (int q = 0; q < MERGE_CHUNK; ++q) M = fmaxf(M, lq[q]);
    float W = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    if (M != -INFINITY) {
#pragma unroll
      for (int q = 0; q < MERGE_CHUNK; ++q) {
        const float w = lq[q] == -INFINITY ? 0.f : exp2f(lq[q] - M);
        W += w;
        acc.x += w * vq[q].x;
        acc.y += w * vq[q].y;
        acc.z += w * vq[q].z;
        acc.w += w * vq[q].w;
      }
    }
    const float inv = W > 0.f ? 1.f / W : 0.f;
    acc.x *= inv;
    acc.y *= inv;
    acc.z *= inv;
    acc.w *= inv;
    if (final_out) {
      uint2 pk;
      pk.x = pack2<T>(acc.x, acc.y);
      pk.y = pack2<T>(acc.z, acc.w);
      *reinterpret_cast<uint2 *>(out + row * D + 4 * cv) = pk;
    } else {
      reinterpret_cast<float4 *>(a.ws2_o + (row * a.max_chunks + dst_idx) * D)[cv] = acc;
      if (cv == 0) a.ws2_lse[row * a.max_chunks + dst_idx] = W > 0.f ? M + log2f(W) : -INFINITY;
    }
  }
}

__device__ __forceinline__ int ld_acquire_gpu(const int32_t *p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Where group tile gt of a work item lies: in the shared span (m = -1; every
// member's tokens, all valid, read through the first member's table), or in
// member m's own span (its tokens from 16*sh on). tok0 is the tile's first
// token in that sequence; len bounds the valid tokens.
struct TileLoc {
  int m, tok0, len;
};

// A warp's register copy of an item's layout: lane i < members holds member
// i's first own tile and length (the lookup below then needs no shared-memory
// reads per tile).
struct ItemView {
  int members, sh, len0, own_r, len_r;
};
__device__ __forceinline__ ItemView item_view(const ItemDesc &d, int lane) {
  ItemView v;
  v.members = d.members;
  v.sh = d.sh;
  v.len0 = d.len[0];
  v.own_r = lane < v.members ? d.own[lane] : INT_MAX;
  v.len_r = lane < v.members ? d.len[lane] : 0;
  return v;
}

// Called by all lanes of a warp with the same gt. GROUPS: the item may attend
// several sequences.
template <bool GROUPS>
__device__ __forceinline__ TileLoc locate_tile(const ItemView &v, int gt, int lane) {
  if (!GROUPS || v.members == 1) return TileLoc{0, gt * TILE, v.len0};  // one sequence
  if (gt < v.sh) return TileLoc{-1, gt * TILE, INT_MAX};
  // own[] is non-decreasing: the member is the number of later members that
  // start at or before gt (lanes past the members hold INT_MAX)
  const int m = __popc(__ballot_sync(FULL_MASK, lane >= 1 && v.own_r <= gt));
  const int own = __shfl_sync(FULL_MASK, v.own_r, m);
  const int len = __shfl_sync(FULL_MASK, v.len_r, m);
  return TileLoc{m, (v.sh + gt - own) * TILE, len};
}

// U8: the block size is an odd multiple of 8, so a 16-token tile is two
// 8-token units that may sit in different blocks.
template <typename T, int D, int NH, bool U8>
__global__ void __launch_bounds__(THREADS, 2)
    decode_tc_kernel(const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const DecodeArgs a) {
  using Shape = TcShape<D, NH>;
  constexpr int NSTAGE = Shape::NSTAGE;
  extern __shared__ uint8_t smem_raw[];
  __shared__ int s_abort;
  const uint32_t raw_addr = smem_addr(smem_raw);
  const uint32_t smem0 = (raw_addr + 1023u) & ~1023u;  // 128B swizzle wants 1024B alignment
  uint8_t *const sm = smem_raw + (smem0 - raw_addr);   // generic view of the same base

  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int Hq = a.num_heads;
  const int Hkv = a.num_kv_heads;
  const int G = Hq / Hkv;
  const int B = a.block_size;

  const uint32_t bars = smem0 + Shape::BAR_OFF;
  auto tile_full = [&](int w, int st) { return bars + 8 * (w * NSTAGE + st); };
  auto item_full = [&](int slot) { return bars + 8 * (NCW * NSTAGE + slot); };
  auto item_empty = [&](int slot) { return bars + 8 * (NCW * NSTAGE + NSLOT + slot); };
  ItemDesc *const desc = reinterpret_cast<ItemDesc *>(sm + Shape::DESC_OFF);
  volatile int *const abort_flag = &s_abort;

  if (threadIdx.x == 0) {
    for (int w = 0; w < NCW; ++w)
      for (int st = 0; st < NSTAGE; ++st) mbar_init(tile_full(w, st), 1);
    for (int sl = 0; sl < NSLOT; ++sl) {
      mbar_init(item_full(sl), 1);
      mbar_init(item_empty(sl), NCW);
    }
    fence_mbar_init();
    prefetch_tensormap(&tmK);
    prefetch_tensormap(&tmV);
    s_abort = 0;
  }
  __syncthreads();
  pdl_wait();  // the work list, counters and everything before the plan are ready

  if (warp == NCW) {
    // ======================= scheduler warp =======================
    // The first item of every CTA is fixed. Its entry lies inside the list's
    // capacity (grid <= capacity x Hkv), so it is loaded together with the
    // list length instead of after it; it is used only if the item exists.
    const uint2 first_wk = a.work[blockIdx.x / Hkv];
    const long long list_cap = (long long)a.num_seqs * a.max_parts;
    const int n_items = (int)min((long long)a.sched[1], list_cap) * Hkv;
    // Tail split (see plan_kernel): items tail_first .. n_items-1 are claimed
    // as tail_split pieces each, so claims run to total_items. (The bounds keep
    // every piece inside the tail region whatever the words hold.)
    int tail_first = n_items, tail_split = 1;
    if (Shape::GROUPS && a.max_group > 1) {  // (the plan wrote the words)
      const int f = a.sched[2], k = a.sched[3];
      if (k >= 2 && k <= TAIL_MAX_SPLIT && f >= (int)gridDim.x && f < n_items &&
          (long long)(n_items - f) * k <= a.tail_slots) {
        tail_first = f;
        tail_split = k;
      }
    }
    const int total_items = tail_first + (n_items - tail_first) * tail_split;
    const int end_phase = total_items - END_ITEMS_PER_CTA * (int)gridDim.x;
    // A CTA that starts after some wait already gave up does no work. The
    // error word is loaded now and checked before the first copy is started,
    // so its latency overlaps the first work-list load.
    const int32_t err_word = (lane == 0 && a.err != nullptr)
                                 ? *reinterpret_cast<volatile const int32_t *>(a.err)
                                 : 0;
    bool first_post = true;
    int item = blockIdx.x;  // the counter starts at grid
    bool claimed = true;  // `item` holds an index taken from the work list
    int in_flight = 0;    // posted work descriptors whose completion is not yet handled
    uint32_t it = 0;      // descriptors posted
    for (;; ++it) {
      const int slot = it % NSLOT;
      ItemDesc &d = desc[slot];
      if (it >= NSLOT) {
        if (!__all_sync(FULL_MASK, wait_or_abort(item_empty(slot), ((it / NSLOT) - 1) & 1,
                                                 abort_flag, a.err)))
          break;
        // The consumers are done with the slot's previous descriptor. A
        // finished partition of a split context is published (a device-scope
        // fence, then a fetch-and-add on its chunk's counter); the warp that
        // completes a chunk merges it here at once, and the one that completes
        // the last chunk merges the chunks into `out`. Merging here, not in
        // the consumers' descriptor stream, keeps the merges from queueing
        // behind the work items already posted.
        const int pk = d.kind;
        if (pk == KIND_WORK) --in_flight;
        const int np = d.nparts;
        if (Shape::GROUPS && pk == KIND_WORK && d.tail >= 0) {
          // a piece of a tail-split item: the warp that completes the item's
          // last piece merges the pieces into `out`
          const int j = d.tail / np;  // the item's first piece slot is j * np
          int t = 0;
          if (lane == 0) {
            __threadfence();
            t = atomicAdd(&a.tail_cnt[j], 1);
          }
          if (__shfl_sync(FULL_MASK, t, 0) == np - 1) {
            (void)ld_acquire_gpu(&a.tail_cnt[j]);  // every lane: the pieces are visible
            merge_range<T, D, true>(a, d.s, d.h, G, d.members, a.tail_o, a.tail_lse, 0, j * np,
                                    j * np + np, true, 0, lane, 32);
          }
        } else if (pk == KIND_WORK && np > 1) {
          const int ms = d.s, mh = d.h, mm = d.members, ch = d.p / MERGE_CHUNK;
          const int nchunks = (np + MERGE_CHUNK - 1) / MERGE_CHUNK;
          int32_t *const cnt1 = &a.merge_cnt[(ms * Hkv + mh) * a.max_chunks + ch];
          int32_t *const cnt2 = &a.merge_cnt2[ms * Hkv + mh];
          int t = 0;
          if (lane == 0) {
            __threadfence();
            t = atomicAdd(cnt1, 1);
          }
          const int ch_size = min(MERGE_CHUNK, np - ch * MERGE_CHUNK);
          if (__shfl_sync(FULL_MASK, t, 0) == ch_size - 1) {
            (void)ld_acquire_gpu(cnt1);  // every lane: the chunk's partials are visible
            bool final_ready = nchunks == 1;
            if (!final_ready) {
              merge_range<T, D>(a, ms, mh, G, mm, a.ws_o, a.ws_lse, a.max_parts,
                                ch * MERGE_CHUNK, ch * MERGE_CHUNK + ch_size, false, ch, lane, 32);
              __threadfence();  // every lane's chunk result precedes the count
              __syncwarp();
              int t2 = 0;
              if (lane == 0) {
                __threadfence();
                t2 = atomicAdd(cnt2, 1);
              }
              final_ready = __shfl_sync(FULL_MASK, t2, 0) == nchunks - 1;
              if (final_ready) (void)ld_acquire_gpu(cnt2);  // the other chunks' results
            }
            if (final_ready) {
              if (nchunks == 1)
                merge_range<T, D>(a, ms, mh, G, mm, a.ws_o, a.ws_lse, a.max_parts, 0, np, true,
                                  0, lane, 32);
              else
                merge_range<T, D>(a, ms, mh, G, mm, a.ws2_o, a.ws2_lse, a.max_chunks, 0, nchunks,
                                  true, 0, lane, 32);
            }
          }
        }
      }
      __syncwarp();  // every lane has read the old descriptor before it is rewritten
      if (!claimed) {
        // End phase: claim the next item only once the descriptor posted two
        // iterations ago is done, so at most two work descriptors are held.
        if (it >= 2) {
          const uint32_t o = it - 2;
          if (!__all_sync(FULL_MASK, wait_or_abort(item_empty(o % NSLOT), (o / NSLOT) & 1,
                                                   abort_flag, a.err)))
            break;
        }
        if (lane == 0) item = atomicAdd(&a.sched[0], 1);
        item = __shfl_sync(FULL_MASK, item, 0);
        claimed = true;
      }
      if (item >= total_items) {
        // No new work: keep the ring turning (no-op descriptors) until every
        // posted item has completed (and its merges are done), then stop.
        if (lane == 0) {
          d.kind = in_flight == 0 ? KIND_END : KIND_NOP;
          d.n_tiles = 0;
          mbar_arrive(item_full(slot));
        }
        if (in_flight == 0) break;
        continue;
      }
      // Before the end phase the next item is claimed now, so that its index
      // is ready when this one has been posted.
      const bool prefetch = item < end_phase;
      int next = 0;
      if (prefetch && lane == 0) next = atomicAdd(&a.sched[0], 1);

      // Items are entry-major: the KV heads of one entry are consecutive items.
      // A block's heads are contiguous in the pool, so CTAs working on
      // neighbouring items read neighbouring 4 KB slices (open DRAM rows).
      // A claim past tail_first is piece `piece` of item `wi` (its pieces are
      // consecutive claims, so they run side by side).
      int wi = item, piece = -1;
      if (Shape::GROUPS && item >= tail_first) {
        const int jj = item - tail_first;
        wi = tail_first + jj / tail_split;
        piece = jj - (jj / tail_split) * tail_split;
      }
      const uint2 wk = first_post ? first_wk : a.work[wi / Hkv];  // first_post: item == blockIdx.x
      const int h = wi - (wi / Hkv) * Hkv;
      const int s = min(static_cast<int>(wk.x >> 16), a.num_seqs - 1);
      const int p = static_cast<int>(wk.x & 0xffffu);
      // One sequence (its clamped length in the entry), or a shared-prefix
      // group led by s (its members' lengths are read here, clamped as the
      // plan clamped them).
      const bool grouped = Shape::GROUPS && (wk.y >> 31) != 0;
      const int members =  // (the plan never forms more; the bounds keep every copy in place)
          grouped ? min((int)((wk.y >> 27) & 15u) + 1,
                        min(min(MAX_MEMBERS, max(1, NH / G)), a.num_seqs - s))
                  : 1;
      const int sh = grouped ? (int)(wk.y & 0x7ffffffu) : 0;
      // Lane m < members: member m's length, own tiles and first own tile.
      // One sequence: its length is the entry's, all its tiles are its own.
      int Lm, own_n, own_lo, tiles;
      if (!grouped) {
        const int L = static_cast<int>(wk.y);
        tiles = (L + TILE - 1) / TILE;
        Lm = lane == 0 ? L : 0;
        own_n = lane == 0 ? tiles : 0;
        own_lo = 0;
      } else {
        Lm = lane < members ? effective_len(a.context_lens[s + lane], a.max_context_len,
                                            a.max_blocks, B, nullptr)
                            : 0;
        own_n = lane < members ? max(0, Lm - sh * TILE + TILE - 1) / TILE : 0;
        int own_incl = own_n;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const int y = __shfl_up_sync(FULL_MASK, own_incl, off);
          if (lane >= off) own_incl += y;
        }
        own_lo = sh + own_incl - own_n;
        tiles = sh + __shfl_sync(FULL_MASK, own_incl, 31);
      }
      // a tail piece: its share of the item's tiles (the plan split only
      // one-partition items)
      const int ptg = piece >= 0 ? max(1, (tiles + tail_split - 1) / tail_split)
                                 : group_part_tiles(a, grouped, tiles);
      const int tile0 = (piece >= 0 ? piece : p) * ptg;
      const int n_tiles = max(0, min(tiles, tile0 + ptg) - tile0);
      if (first_post) {
        first_post = false;
        if (__shfl_sync(FULL_MASK, err_word == PKV_DEV_WAIT_TIMEOUT ? 1 : 0, 0)) {
          if (lane == 0) *abort_flag = 1;  // the consumers' waits see it and stop
          break;
        }
      }
      // The members' q rows (and, with one sequence per item, the newest
      // token's K and V rows of a fused append) are copied first: the copies
      // complete on the slot's barrier while the lanes fetch the block ids,
      // and the arrival that publishes the descriptor comes last.
      const uint32_t qbytes = n_tiles > 0 ? (uint32_t)(G * D * 2) : 0u;
      const uint32_t stage = smem0 + Shape::QBUF_OFF + slot * Shape::QBUF_BYTES;
      if (!grouped) {  // one sequence: lane 0 issues everything
        const int last = own_n - 1;       // its last tile holds token L-1
        const uint32_t rbytes =
            a.k_new != nullptr && last >= tile0 && last < tile0 + n_tiles ? (uint32_t)(D * 2) : 0u;
        if (lane == 0) {
          mbar_expect_tx(item_full(slot), qbytes + 2 * rbytes);
          if (qbytes)
            bulk_load(stage, static_cast<const T *>(a.q) + ((size_t)s * Hq + h * G) * D, qbytes,
                      item_full(slot));
          if (rbytes) {
            const size_t row = ((size_t)s * Hkv + h) * D;
            bulk_load(stage + Shape::QROWS_BYTES, static_cast<const T *>(a.k_new) + row, rbytes,
                      item_full(slot));
            bulk_load(stage + Shape::QROWS_BYTES + D * 2, static_cast<const T *>(a.v_new) + row,
                      rbytes, item_full(slot));
          }
        }
      } else {
        if (lane == 0) mbar_expect_tx(item_full(slot), members * qbytes);
        __syncwarp();  // the expected bytes are set before any copy can complete
        if (lane < members && qbytes)
          bulk_load(stage + lane * qbytes,
                    static_cast<const T *>(a.q) + ((size_t)(s + lane) * Hq + h * G) * D, qbytes,
                    item_full(slot));
      }
      constexpr int upt = U8 ? 2 : 1;  // table entries per tile
      // All of a lane's table loads are issued before its first store.
      int idv[IDS_PER_LANE];
      if (!grouped) {  // one sequence: partition tile t is its tile tile0 + t
        const int L = static_cast<int>(wk.y);
        const int32_t *bt = a.block_tables + (size_t)s * a.max_blocks;
#pragma unroll
        for (int k = 0; k < IDS_PER_LANE; ++k) {
          const int t = lane + 32 * k;
          const int tok = tile0 * TILE + t * (TILE / upt);
          idv[k] = t < n_tiles * upt && tok < L ? bt[tok / B] : -1;  // none read past the context
        }
      } else {
        // Member m's first own tile and length in every lane (for the lookup).
        int own_v[MAX_MEMBERS], len_v[MAX_MEMBERS];
#pragma unroll
        for (int m = 0; m < MAX_MEMBERS; ++m) {
          own_v[m] = __shfl_sync(FULL_MASK, own_lo, m);
          len_v[m] = __shfl_sync(FULL_MASK, Lm, m);
        }
#pragma unroll
        for (int k = 0; k < IDS_PER_LANE; ++k) {
          const int t = lane + 32 * k;
          const int gt = tile0 + t / upt;  // group tile
          int m = 0, first = own_v[0], len = len_v[0];  // (selected without dynamic indexing)
          if (gt >= sh) {  // a member's own tile
#pragma unroll
            for (int i = 1; i < MAX_MEMBERS; ++i)
              if (i < members && own_v[i] <= gt) {
                m = i;
                first = own_v[i];
                len = len_v[i];
              }
          }
          const int tok = (gt >= sh ? sh + gt - first : gt) * TILE + (t % upt) * (TILE / upt);
          // none read past the context
          idv[k] = t < n_tiles * upt && tok < len
                       ? a.block_tables[(size_t)(s + m) * a.max_blocks + tok / B]
                       : -1;
        }
      }
#pragma unroll
      for (int k = 0; k < IDS_PER_LANE; ++k)
        if (lane + 32 * k < n_tiles * upt) d.ids[lane + 32 * k] = idv[k];
      if (lane < members) {
        d.own[lane] = own_lo;
        d.len[lane] = Lm;
      }
      if (lane == 0) {
        d.kind = KIND_WORK;
        d.s = s;
        d.p = piece >= 0 ? piece : p;
        d.h = h;
        d.n_tiles = n_tiles;
        d.nparts = piece >= 0 ? tail_split : (tiles + ptg - 1) / ptg;
        if constexpr (Shape::GROUPS) d.tail = piece >= 0 ? item - tail_first : -1;
        d.members = members;
        d.tile0 = tile0;
        d.sh = sh;
        d.own[members] = tiles;
      }
      __syncwarp();  // every lane's ids precede lane 0's release below
      if (lane == 0) mbar_arrive(item_full(slot));
      ++in_flight;
      if (prefetch)
        item = __shfl_sync(FULL_MASK, next, 0);
      else
        claimed = false;
    }
    // After a stop, the q copies of the last descriptors posted may still be
    // landing in shared memory: wait for them (bounded) before leaving.
    if (*abort_flag)
      for (uint32_t k = it > NSLOT ? it - NSLOT : 0; k < it; ++k)
        wait_bounded(item_full(k % NSLOT), (k / NSLOT) & 1);
    // This CTA posts nothing more: the next call's grids may start launching
    // (they wait for this grid to complete before touching memory).
    if (lane == 0) pdl_launch_dependents();
    return;
  }

  // ======================= consumer warps =======================
  const int g = lane >> 2;  // mma group id (row of A / column of B)
  const int c = lane & 3;   // thread in group
  // Members owning this lane's score columns 2c, 2c+1 (column n is member n / G).
  const int mc0 = (2 * c) / G, mc1 = (2 * c + 1) / G;
  const float sl2 = a.scale_log2;
  T *const out = static_cast<T *>(a.out);
  const int mi = lane >> 3;                      // ldmatrix: lane feeds row (lane & 7)
  const int vr = (lane & 7) + ((mi >> 1) << 3);  //   of matrix mi; token row in the tile
  constexpr int AS = Shape::ACC_STRIDE;
  const uint32_t ring = smem0 + warp * NSTAGE * Shape::STAGE_BYTES;
  const int total_rows = a.num_blocks * Hkv * B;
  float *const scales = reinterpret_cast<float *>(sm + Shape::SCALES_OFF);  // [NH][NCW], [NH]
  int *const comb_stage = reinterpret_cast<int *>(scales + NH * (NCW + 1));  // [NCW]
  constexpr int CH = D / 8;                 // 16-byte chunks per K or V row
  const int e_ch = lane % CH, kv_ch = lane / CH;  // fused append: lanes < CH K, < 2CH V

  // Issue side of this warp's ring. It walks the same descriptor sequence as
  // the consume side but runs up to NSTAGE tiles ahead, across item boundaries.
  uint32_t issued = 0, done = 0;  // tiles of this warp issued / consumed so far
  uint32_t bad_mask = 0;          // bit st: the tile in stage st had an invalid block id
  uint32_t is_it = 0;             // descriptor being issued
  int is_j = 0, is_ntw = 0, is_h = 0, is_tile0 = 0, is_s = 0;
  ItemView is_view{1, 0, 0, 0, 0};
  bool is_ready = false, is_end = false;

  // Issue this warp's next tiles while fewer than NSTAGE are in flight. With
  // `must`, block (bounded) for the next descriptor when nothing is in flight.
  auto pump = [&](bool must) {
    while (issued - done < (uint32_t)NSTAGE && !is_end) {
      if (!is_ready) {
        const int sl = is_it % NSLOT;
        const uint32_t par = (is_it / NSLOT) & 1;
        bool ok;
        if (must && issued == done)
          ok = wait_or_abort(item_full(sl), par, abort_flag, a.err);
        else
          ok = mbar_test(item_full(sl), par);
        if (!__all_sync(FULL_MASK, ok)) return;
        const ItemDesc &d = desc[sl];
        if (d.kind == KIND_END) {
          is_end = true;
          return;
        }
        const int nt = d.kind == KIND_WORK ? d.n_tiles : 0;
        is_s = d.s;
        is_h = d.h;
        is_tile0 = d.tile0;
        is_view = item_view(d, lane);
        is_ntw = warp < nt ? (nt - warp + NCW - 1) / NCW : 0;
        is_j = 0;
        is_ready = true;
      }
      if (is_j >= is_ntw) {
        ++is_it;
        is_ready = false;
        continue;
      }
      const int tile = warp + is_j * NCW;
      const ItemDesc &dd = desc[is_it % NSLOT];
      const TileLoc loc = locate_tile<Shape::GROUPS>(is_view, is_tile0 + tile, lane);
      const int tok0 = loc.tok0;
      const size_t trow =  // its table row
          (size_t)(Shape::GROUPS ? is_s + max(loc.m, 0) : is_s) * a.max_blocks;
      const int st = issued % NSTAGE;
      // Pool row of each unit of the tile. total_rows is wholly out of
      // bounds, and TMA fills zeros there. It is used for an invalid block id,
      // which is reported, and for a second unit past the context, whose
      // table entry is not read. The first unit always starts before the end
      // of its sequence.
      constexpr int upt = U8 ? 2 : 1;
      const int idx0 = tile * upt;
      const int p0 = idx0 < DESC_IDS ? dd.ids[idx0] : a.block_tables[trow + tok0 / B];
      bool bad = p0 < 0 || p0 >= a.num_blocks;
      const int y0 = bad ? total_rows : (p0 * Hkv + is_h) * B + (tok0 % B);
      int y1 = total_rows;
      if (U8 && tok0 + TILE / 2 < loc.len) {
        const int tok1 = tok0 + TILE / 2;
        const int p1 = idx0 + 1 < DESC_IDS ? dd.ids[idx0 + 1] : a.block_tables[trow + tok1 / B];
        const bool bad1 = p1 < 0 || p1 >= a.num_blocks;
        bad = bad || bad1;
        if (!bad1) y1 = (p1 * Hkv + is_h) * B + (tok1 % B);
      }
      bad_mask = bad ? (bad_mask | (1u << st)) : (bad_mask & ~(1u << st));
      if (lane == 0) {
        if (bad) report(a.err, PKV_DEV_BAD_BLOCK);
        const uint32_t bar = tile_full(warp, st);
        const uint32_t kdst = ring + st * Shape::STAGE_BYTES;
        const uint32_t vdst = kdst + Shape::KT_BYTES;
        mbar_arrive_expect_tx(bar, Shape::STAGE_BYTES);
        if constexpr (U8) {
          // two 8-row boxes per 64-element half (2D map): rows 0-7 and 8-15
#pragma unroll
          for (int hh = 0; hh < Shape::HALVES; ++hh) {
            const uint32_t o = hh * HALF_BYTES;
            tma_load_2d(kdst + o, &tmK, hh * BOX_COLS, y0, bar);
            tma_load_2d(kdst + o + HALF_BYTES / 2, &tmK, hh * BOX_COLS, y1, bar);
            tma_load_2d(vdst + o, &tmV, hh * BOX_COLS, y0, bar);
            tma_load_2d(vdst + o + HALF_BYTES / 2, &tmV, hh * BOX_COLS, y1, bar);
          }
        } else if constexpr (Shape::HALVES == 1) {
          tma_load_2d(kdst, &tmK, 0, y0, bar);
          tma_load_2d(vdst, &tmV, 0, y0, bar);
        } else {  // both halves of the tile in one copy each (3D map)
          tma_load_3d(kdst, &tmK, 0, y0, 0, bar);
          tma_load_3d(vdst, &tmV, 0, y0, 0, bar);
        }
      }
      ++issued;
      ++is_j;
    }
  };

  bool stop = false;  // a wait of this warp gave up during the previous item
  for (uint32_t it = 0;; ++it) {
    const int slot = it % NSLOT;
    const bool got = wait_or_abort(item_full(slot), (it / NSLOT) & 1, abort_flag, a.err);
    // One vote per item. All consumers have finished the previous item (its
    // combine-area reads included) before any passes, and all take the same
    // exit decision.
    if (!consumers_all(got && !stop && *abort_flag == 0)) break;
    const ItemDesc &dref = desc[slot];
    const int kind = dref.kind;
    if (kind == KIND_END) break;  // the same descriptor for every consumer: a uniform exit
    if (kind != KIND_WORK) {  // a no-op that keeps the ring turning
      pump(false);
      consumers_sync();  // the descriptor is read by all before the slot is handed back
      if (lane == 0) mbar_arrive(item_empty(slot));
      continue;
    }
    const int s = dref.s, p = dref.p, h = dref.h, n_tiles = dref.n_tiles;
    const int nparts = dref.nparts, tail = Shape::GROUPS ? dref.tail : -1;
    const int members = dref.members, tile0 = dref.tile0;
    const bool one_seq = !Shape::GROUPS || members == 1;
    const int ncol = members * G;  // head rows attended: G per member
    // this lane's two columns (query heads 2c, 2c+1 of the rows) belong to these members
    const bool col0_live = mc0 < members, col1_live = mc1 < members;
    const int nt_w = warp < n_tiles ? (n_tiles - warp + NCW - 1) / NCW : 0;

    pump(false);  // top up the ring (this item, and beyond)

    // Q^T as the B operand: lane (g, c) holds head g's elements
    // 8*Lc .. 8*Lc+7 for logical chunk Lc(c, j) = (j/2)*8 + 2c + (j%2).
    uint4 qf[D / 32];
    {
      const uint32_t qrow = smem0 + Shape::QBUF_OFF + slot * Shape::QBUF_BYTES + g * D * 2;
#pragma unroll
      for (int j = 0; j < D / 32; ++j) {
        const int Lc = (j >> 1) * 8 + 2 * c + (j & 1);
        qf[j] = (g < ncol && n_tiles > 0) ? lds128(qrow + Lc * 16) : make_uint4(0, 0, 0, 0);
      }
    }

    float acc[D / 16][4];
#pragma unroll
    for (int mt = 0; mt < D / 16; ++mt) acc[mt][0] = acc[mt][1] = acc[mt][2] = acc[mt][3] = 0.f;
    float m0 = -INFINITY, m1 = -INFINITY;  // reference max of heads 2c, 2c+1 (base-2 units)
    float l0 = 0.f, l1 = 0.f;              // this lane's share of the running sums
    bool aborted = false;
    // Combine rows: `rows` columns per warp, in the combine area or (held) in
    // the ring stage of the warp's last tile of the item (last_st).
    const bool held = Shape::RING_COMBINE && ncol > Shape::SMALL_COLS;
    const int rows = held || !Shape::RING_COMBINE ? NH : Shape::SMALL_COLS;
    int last_st = -1;

    const ItemView view = item_view(dref, lane);
    const int L0 = view.len0;  // one sequence: its length
    // Fused append, one sequence: the j of this warp's tile that holds token L-1.
    int j_new = -1;
    if (a.k_new != nullptr && one_seq && L0 > 0) {
      const int idx = (L0 - 1) / TILE - tile0;
      if (idx >= 0 && idx < n_tiles && idx % NCW == warp) j_new = idx / NCW;
    }
    // Fused append, a group: the K (lanes < CH) or V (lanes CH..2CH-1) row
    // chunk of the newest token of the member whose last tile is this warp's
    // j-th tile, read from k_new / v_new one tile before it is used.
    auto fetch_newest = [&](int j) {
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if constexpr (Shape::GROUPS) {
        // (one sequence: its rows were staged with its q rows)
        if (a.k_new == nullptr || one_seq || j >= nt_w) return v;  // (uniform)
        const TileLoc l = locate_tile<Shape::GROUPS>(view, tile0 + warp + j * NCW, lane);
        if (l.m < 0 || l.len - 1 >= l.tok0 + TILE || lane >= 2 * CH) return v;
        const T *src = static_cast<const T *>(kv_ch ? a.v_new : a.k_new) +
                       ((size_t)(s + l.m) * Hkv + h) * D + e_ch * 8;
        v = __ldg(reinterpret_cast<const uint4 *>(src));
      }
      return v;
    };
    // The tile loop, compiled once for one sequence per item (GRP false: plain
    // tile arithmetic) and once for a group (shared and own tiles).
    auto run_tiles = [&](auto grp_tag) {
    constexpr bool GRP = decltype(grp_tag)::value;
    uint4 newest = GRP ? fetch_newest(0) : make_uint4(0u, 0u, 0u, 0u);
    for (int j = 0; j < nt_w; ++j) {
      const uint4 newest_next = GRP ? fetch_newest(j + 1) : make_uint4(0u, 0u, 0u, 0u);
      if (issued == done) pump(true);
      const int st = done % NSTAGE;
      if (issued == done ||
          !__all_sync(FULL_MASK, wait_or_abort(tile_full(warp, st), (done / NSTAGE) & 1,
                                               abort_flag, a.err))) {
        aborted = true;
        break;
      }
      const uint32_t ks = ring + st * Shape::STAGE_BYTES;
      const uint32_t vs = ks + Shape::KT_BYTES;
      const int tile_idx = warp + j * NCW;
      const bool bad = (bad_mask >> st) & 1u;
      // Where the tile lies. A shared tile counts for every member's columns,
      // an own tile for its member's only.
      int tok0, valid, mem, len;  // mem = -1: shared
      bool use0, use1, has_new;
      if constexpr (!GRP) {
        tok0 = (tile0 + tile_idx) * TILE;
        len = L0;
        valid = min(TILE, L0 - tok0);
        mem = 0;
        use0 = true;  // columns past the G heads hold zero queries and are never combined
        use1 = true;
        has_new = j == j_new;
      } else {
        const TileLoc loc = locate_tile<Shape::GROUPS>(view, tile0 + tile_idx, lane);
        tok0 = loc.tok0;
        len = loc.len;
        mem = loc.m;
        valid = mem < 0 ? TILE : min(TILE, len - tok0);
        use0 = mem < 0 ? col0_live : mc0 == mem;
        use1 = mem < 0 ? col1_live : mc1 == mem;
        has_new = a.k_new != nullptr && mem >= 0 && len - 1 < tok0 + TILE;
      }

      if (has_new && !bad) {
        // Fused append: this tile holds token L-1 of member mem. Its K and V
        // rows come from the new rows (whatever the pool slot held), and the
        // same rows are written to the pool slot: that is the cache-append.
        const int r = len - 1 - tok0;
        const int e = e_ch, kv = kv_ch;
        if (lane < 2 * CH) {
          uint4 v;
          if constexpr (!GRP)
            v = lds128(smem0 + Shape::QBUF_OFF + slot * Shape::QBUF_BYTES + Shape::QROWS_BYTES +
                       kv * D * 2 + e * 16);
          else
            v = newest;
          const uint32_t tile_base = kv ? vs : ks;
          sts128(tile_base + (e >> 3) * HALF_BYTES + r * 128 + (((e & 7) ^ (r & 7)) << 4), v);
          const int tok = len - 1;
          const int idx = U8 ? tile_idx * 2 + (r >> 3) : tile_idx;
          const int blk = idx < DESC_IDS
                              ? desc[slot].ids[idx]
                              : a.block_tables[(size_t)(s + mem) * a.max_blocks + tok / B];
          T *pool = static_cast<T *>(const_cast<void *>(kv ? a.v_pool : a.k_pool));
          *reinterpret_cast<uint4 *>(pool + (((size_t)blk * Hkv + h) * B + tok % B) * D + e * 8) = v;
        }
        fence_proxy_async_smem();  // these writes precede the stage's next TMA fill
        __syncwarp();
      }
      if (valid < TILE && !bad) {
        // Tokens past the context length: their V rows may hold anything
        // (NaN included); zero them so P*V stays finite.
        const int nchunks = (TILE - valid) * 8 * Shape::HALVES;
        for (int e = lane; e < nchunks; e += 32) {
          const int r = valid + e / (8 * Shape::HALVES);
          const int rem = e % (8 * Shape::HALVES);
          sts128_zero(vs + (rem >> 3) * HALF_BYTES + r * 128 + (rem & 7) * 16);
        }
        fence_proxy_async_smem();  // these writes precede the stage's next TMA fill
        __syncwarp();
      }

      // ---- scores: S^T = K . Q^T in independent accumulation chains: two
      // (sa, sb), and with 4 columns two more (sc, sd) for the odd k-chunks.
      // (Four chains in the 8-column layout measured 5-6 % slower.) ----
      float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f};
      if constexpr (Shape::GROUPS) {
#pragma unroll
        for (int jj = 0; jj < D / 32; ++jj) {
          const int Lc = (jj >> 1) * 8 + 2 * c + (jj & 1);
          const uint32_t rowg = ks + (Lc >> 3) * HALF_BYTES + g * 128 + (((Lc & 7) ^ g) << 4);
          const uint4 ka = lds128(rowg);            // token g
          const uint4 kb = lds128(rowg + 8 * 128);  // token g + 8 (same swizzle phase)
          mma16816<T>(sa, ka.x, kb.x, ka.y, kb.y, qf[jj].x, qf[jj].y);
          mma16816<T>(sb, ka.z, kb.z, ka.w, kb.w, qf[jj].z, qf[jj].w);
        }
      } else {
        float sc[4] = {0.f, 0.f, 0.f, 0.f}, sd[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int jj = 0; jj < D / 32; ++jj) {
          const int Lc = (jj >> 1) * 8 + 2 * c + (jj & 1);
          const uint32_t rowg = ks + (Lc >> 3) * HALF_BYTES + g * 128 + (((Lc & 7) ^ g) << 4);
          const uint4 ka = lds128(rowg);            // token g
          const uint4 kb = lds128(rowg + 8 * 128);  // token g + 8 (same swizzle phase)
          if (jj & 1) {
            mma16816<T>(sc, ka.x, kb.x, ka.y, kb.y, qf[jj].x, qf[jj].y);
            mma16816<T>(sd, ka.z, kb.z, ka.w, kb.w, qf[jj].z, qf[jj].w);
          } else {
            mma16816<T>(sa, ka.x, kb.x, ka.y, kb.y, qf[jj].x, qf[jj].y);
            mma16816<T>(sb, ka.z, kb.z, ka.w, kb.w, qf[jj].z, qf[jj].w);
          }
        }
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          sa[r] += sc[r];
          sb[r] += sd[r];
        }
      }

      // ---- online softmax (heads 2c, 2c+1; tokens g, g+8) ----
      const bool ok0 = !bad && g < valid;
      const bool ok1 = !bad && g + 8 < valid;
      const float x0 = ok0 && use0 ? (sa[0] + sb[0]) * sl2 : -INFINITY;
      const float x1 = ok0 && use1 ? (sa[1] + sb[1]) * sl2 : -INFINITY;
      const float x2 = ok1 && use0 ? (sa[2] + sb[2]) * sl2 : -INFINITY;
      const float x3 = ok1 && use1 ? (sa[3] + sb[3]) * sl2 : -INFINITY;
      float mx0 = fmaxf(x0, x2), mx1 = fmaxf(x1, x3);
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) {
        mx0 = fmaxf(mx0, __shfl_xor_sync(FULL_MASK, mx0, off));
        mx1 = fmaxf(mx1, __shfl_xor_sync(FULL_MASK, mx1, off));
      }
      // Lazy reference max: keep it unless this tile exceeds it by more than
      // 2^RESCALE_SLACK (then p <= 2^8 stays well inside fp32/bf16/fp16 range).
      const bool up0 = mx0 > m0 + RESCALE_SLACK, up1 = mx1 > m1 + RESCALE_SLACK;
      if (__any_sync(FULL_MASK, up0 || up1)) {
        const float mn0 = up0 ? mx0 : m0, mn1 = up1 ? mx1 : m1;
        const float al0 = m0 == -INFINITY ? 0.f : ex2_approx(m0 - mn0);
        const float al1 = m1 == -INFINITY ? 0.f : ex2_approx(m1 - mn1);
        l0 *= al0;
        l1 *= al1;
#pragma unroll
        for (int mt = 0; mt < D / 16; ++mt) {
          acc[mt][0] *= al0;
          acc[mt][1] *= al1;
          acc[mt][2] *= al0;
          acc[mt][3] *= al1;
        }
        m0 = mn0;
        m1 = mn1;
      }
      const float mu0 = m0 == -INFINITY ? 0.f : m0;
      const float mu1 = m1 == -INFINITY ? 0.f : m1;
      const float p0 = ex2_approx(x0 - mu0), p1 = ex2_approx(x1 - mu1);
      const float p2 = ex2_approx(x2 - mu0), p3 = ex2_approx(x3 - mu1);
      l0 += p0 + p2;
      l1 += p1 + p3;

      // P^T as the B operand: transpose the (token, head) fragment pairs.
      // The tensor core takes P in the input type. One bf16 rounding (up to
      // 2^-8 relative per weight) can exceed the accuracy bound when value
      // rows nearly cancel, so for bf16 P is carried as hi + lo (about 16
      // bits). For fp16 one rounding (2^-11) bounds the output error by
      // 2^-11 * max|v|, inside the bound, and P stays a single operand.
      const uint32_t w01 = pack2<T>(p0, p1), w23 = pack2<T>(p2, p3);
      const uint32_t pb0 = movmatrix_trans(w01);  // tokens 0..7
      const uint32_t pb1 = movmatrix_trans(w23);  // tokens 8..15
      constexpr bool kSplitP = std::is_same<T, __nv_bfloat16>::value;
      [[maybe_unused]] uint32_t pl0 = 0, pl1 = 0;
      if constexpr (kSplitP) {
        pl0 = movmatrix_trans(pack2<T>(p0 - lo_half_to_float<T>(w01), p1 - hi_half_to_float<T>(w01)));
        pl1 = movmatrix_trans(pack2<T>(p2 - lo_half_to_float<T>(w23), p3 - hi_half_to_float<T>(w23)));
      }

      // ---- O^T += V^T . P^T ----
      const uint32_t vrow = vs + vr * 128;
#pragma unroll
      for (int mt = 0; mt < D / 16; ++mt) {
        const int chunk = 2 * mt + (mi & 1);
        const uint32_t addr = vrow + (chunk >> 3) * HALF_BYTES + (((chunk & 7) ^ (vr & 7)) << 4);
        uint32_t r0, r1, r2, r3;
        ldsm_x4_trans(addr, r0, r1, r2, r3);
        mma16816<T>(acc[mt], r0, r1, r2, r3, pb0, pb1);
        if constexpr (kSplitP) mma16816<T>(acc[mt], r0, r1, r2, r3, pl0, pl1);
      }
      __syncwarp();  // every lane is done with this stage before it is refilled
      ++done;
      newest = newest_next;
      if (held && j + 1 == nt_w)
        last_st = st;  // it takes this warp's combine rows; refilled after the next vote
      else
        pump(false);
    }
    };
    if (Shape::GROUPS && !one_seq)
      run_tiles(std::true_type{});
    else
      run_tiles(std::false_type{});

    // Full per-warp sums: add the 8 lanes that share a head pair.
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      l0 += __shfl_xor_sync(FULL_MASK, l0, off);
      l1 += __shfl_xor_sync(FULL_MASK, l1, off);
    }

    // ---- combine the consumer warps ----
    // 1) each warp stores its unnormalised rows and (max, sum) per column:
    //    into its own combine area, or (held) into the stage of its last
    //    tile, where a warp without tiles stores nothing
    const int cw_floats = rows * AS + 2 * rows;
    float *const own_area = reinterpret_cast<float *>(sm + Shape::COMBINE_OFF);
    float *cw = nullptr;
    if (held) {
      if (last_st >= 0)
        cw = reinterpret_cast<float *>(sm + (size_t)(warp * NSTAGE + last_st) *
                                                Shape::STAGE_BYTES);
    } else {
      cw = own_area + warp * cw_floats;
    }
    if (cw != nullptr) {
#pragma unroll
      for (int mt = 0; mt < D / 16; ++mt) {
        if (2 * c < rows) {
          cw[(2 * c) * AS + 16 * mt + g] = acc[mt][0];
          cw[(2 * c) * AS + 16 * mt + g + 8] = acc[mt][2];
        }
        if (2 * c + 1 < rows) {
          cw[(2 * c + 1) * AS + 16 * mt + g] = acc[mt][1];
          cw[(2 * c + 1) * AS + 16 * mt + g + 8] = acc[mt][3];
        }
      }
      if (g == 0) {
        if (2 * c < rows) {
          cw[rows * AS + 2 * c] = m0;
          cw[rows * AS + rows + 2 * c] = l0;
        }
        if (2 * c + 1 < rows) {
          cw[rows * AS + 2 * c + 1] = m1;
          cw[rows * AS + rows + 2 * c + 1] = l1;
        }
      }
      if (held) fence_proxy_async_smem();  // these writes precede the stage's next TMA fill
    }
    if (held && lane == 0) comb_stage[warp] = last_st;
    consumers_sync();
    const float *area[NCW];  // each warp's combine rows, or null
#pragma unroll
    for (int w = 0; w < NCW; ++w) {
      if (held) {
        const int st = comb_stage[w];
        area[w] = st < 0 ? nullptr
                         : reinterpret_cast<const float *>(
                               sm + (size_t)(w * NSTAGE + st) * Shape::STAGE_BYTES);
      } else {
        area[w] = own_area + w * cw_floats;
      }
    }
    // 2) per column: warp weights 2^(m_w - M) / sum, and the log2-sum-exp
    if (threadIdx.x < ncol) {
      const int n = threadIdx.x;
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < NCW; ++w)
        if (area[w]) M = fmaxf(M, area[w][rows * AS + n]);
      float f[NCW], den = 0.f;
#pragma unroll
      for (int w = 0; w < NCW; ++w) {
        const float mw = area[w] ? area[w][rows * AS + n] : -INFINITY;
        f[w] = (M == -INFINITY || mw == -INFINITY) ? 0.f : ex2_approx(mw - M);
        if (area[w]) den += f[w] * area[w][rows * AS + rows + n];
      }
      const float inv = den > 0.f ? 1.f / den : 0.f;
#pragma unroll
      for (int w = 0; w < NCW; ++w) scales[n * NCW + w] = f[w] * inv;
      scales[NH * NCW + n] = den > 0.f ? M + lg2_approx(den) : -INFINITY;
    }
    consumers_sync();
    // 3) outputs: element dd of column n's combined row
    auto combined = [&](int n, int dd) {
      float o = 0.f;
#pragma unroll
      for (int w = 0; w < NCW; ++w)
        if (area[w]) o += scales[n * NCW + w] * area[w][n * AS + dd];
      return o;
    };
    if (tail >= 0) {  // a tail piece: column n goes to row n of its slot
      for (int idx = threadIdx.x; idx < ncol * D; idx += NCW * 32) {
        const int n = idx / D;
        const int dd = idx - n * D;
        a.tail_o[((size_t)tail * TAIL_COLS + n) * D + dd] = combined(n, dd);
        if (dd == 0) a.tail_lse[(size_t)tail * TAIL_COLS + n] = scales[NH * NCW + n];
      }
    } else {
      const bool single = nparts <= 1;
      for (int idx = threadIdx.x; idx < ncol * D; idx += NCW * 32) {
        const int n = idx / D;
        const int dd = idx - n * D;
        const float o = combined(n, dd);
        const int mem = n / G;  // row n is query head h*G + n%G of member mem
        const size_t row = (size_t)(s + mem) * Hq + h * G + (n - mem * G);
        if (single) {
          out[row * D + dd] = from_float<T>(o);
        } else {
          a.ws_o[(row * a.max_parts + p) * D + dd] = o;
          if (dd == 0) a.ws_lse[row * a.max_parts + p] = scales[NH * NCW + n];
        }
      }
    }
    // This warp is done with the item's descriptor and q rows. Its arrival
    // (after the warp's lanes have synchronised) hands the slot back and
    // publishes the warp's global writes to the scheduler.
    __syncwarp();
    if (lane == 0) mbar_arrive(item_empty(slot));
    stop = aborted;
  }

  // After a stop, copies this warp issued may still be landing in its ring:
  // wait for them (bounded) before the CTA's shared memory is released.
  for (; done != issued; ++done)
    if (!__all_sync(FULL_MASK, wait_bounded(tile_full(warp, done % NSTAGE), (done / NSTAGE) & 1)))
      break;
}

int sm_count_for_current_device() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    return 148;
  return n;
}

template <typename T, int D, int NH, bool U8>
cudaError_t launch_tc(const DecodeArgs &a, const CUtensorMap &tmK, const CUtensorMap &tmV,
                      cudaStream_t stream) {
  using Shape = TcShape<D, NH>;
  auto kern = decode_tc_kernel<T, D, NH, U8>;
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Shape::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, THREADS, Shape::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) per_sm = 1;
  const long long max_items = (long long)a.num_seqs * a.max_parts * a.num_kv_heads;
  long long grid = (long long)sm_count_for_current_device() * per_sm;
  if (grid > max_items) grid = max_items;
  if (grid < 1) grid = 1;
  DecodeArgs b = a;
  b.grid = (int)grid;
  // With 8 columns, rows left over by one sequence's G query heads are filled
  // with the heads of further sequences that share a prefix with it (up to
  // 8 / G of them); with 4 columns an item attends one sequence.
  const int groups_of = NH / (a.num_heads / a.num_kv_heads);
  b.max_group = Shape::GROUPS ? max(1, min(MAX_MEMBERS, groups_of)) : 1;

  // Both launches are programmatic dependents of what precedes them in the
  // stream. The plan may start while a previous decode call finishes (it
  // waits for that call before touching memory); the decode CTAs start
  // (barrier set-up, descriptor prefetch) while the plan runs, and wait for
  // it before reading the work list.
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t pcfg = {};
  pcfg.gridDim = dim3(1);
  pcfg.blockDim = dim3(PLAN_THREADS);
  pcfg.dynamicSmemBytes = 0;
  pcfg.stream = stream;
  pcfg.attrs = attr;
  pcfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&pcfg, plan_kernel<Shape::GROUPS>, b);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(THREADS);
  cfg.dynamicSmemBytes = Shape::SMEM_BYTES;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, tmK, tmV, b);
}

template <typename T, bool U8>
cudaError_t launch_tc_t(const DecodeArgs &a, const CUtensorMap &tmK, const CUtensorMap &tmV,
                        cudaStream_t stream) {
  // 4 score columns for 3 or 4 query heads per KV head (one sequence per
  // item). Otherwise 8: the G heads of one sequence, or with G = 1, 2 the
  // heads of up to 8 / G sequences that share a prefix.
  const int G = a.num_heads / a.num_kv_heads;
  const bool four = G == 3 || G == 4;
  if (a.head_dim == 64)
    return four ? launch_tc<T, 64, 4, U8>(a, tmK, tmV, stream)
                : launch_tc<T, 64, 8, U8>(a, tmK, tmV, stream);
  return four ? launch_tc<T, 128, 4, U8>(a, tmK, tmV, stream)
              : launch_tc<T, 128, 8, U8>(a, tmK, tmV, stream);
}

}  // namespace

size_t decode_tc_smem_bytes(int head_dim) {
  return head_dim == 64 ? TcShape<64, 8>::SMEM_BYTES : TcShape<128, 8>::SMEM_BYTES;
}

cudaError_t launch_wait_timeout_probe(long long limit_cycles, int32_t *err, cudaStream_t stream) {
  wait_timeout_probe_kernel<<<1, 32, 0, stream>>>(limit_cycles, err);
  return cudaGetLastError();
}

cudaError_t launch_decode_tc(const DecodeArgs &a, int dtype, const CUtensorMap &tmK,
                             const CUtensorMap &tmV, cudaStream_t stream) {
  if (dtype == PKV_BF16)
    return a.unit8 ? launch_tc_t<__nv_bfloat16, true>(a, tmK, tmV, stream)
                   : launch_tc_t<__nv_bfloat16, false>(a, tmK, tmV, stream);
  return a.unit8 ? launch_tc_t<__half, true>(a, tmK, tmV, stream)
                 : launch_tc_t<__half, false>(a, tmK, tmV, stream);
}

}  // namespace pkv
