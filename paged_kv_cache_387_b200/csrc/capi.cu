// C ABI entry points: argument checks, workspace layout, TMA descriptors and
// launches. No allocation happens here. Every buffer belongs to the caller.
#include <cudaTypedefs.h>
#include <math.h>
#include <stdint.h>

#include <atomic>
#include <mutex>

#include "pkv.h"
#include "pkv_internal.h"

namespace {

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Partitions needed for the longest allowed context (1 when unsplit).
long long parts_for(int max_context_len, int partition_size) {
  if (partition_size <= 0) return 1;
  const long long L = max_context_len > 0 ? max_context_len : 1;
  return (L + partition_size - 1) / partition_size;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_tiled_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// A pool viewed as a 2-D tensor [rows = num_blocks*Hkv*B][D] of 16-bit
// elements. It is read in boxes of 64 elements x 16 rows under the 128-byte
// swizzle.
// The pool as rows of head_dim 16-bit elements. A 128-byte swizzled box row
// holds 64 elements, so a row of head_dim = 128 is two 64-element halves. For
// that case the map is 3D, {64 elements, rows, halves}, with the halves
// 128 bytes apart: one box {64, 16, 2} then lands as [half][16 rows][128 B],
// a whole 16-token tile in one copy. head_dim = 64 uses the 2D map {64, rows}.
bool make_pool_map(CUtensorMap *map, const void *pool, long long rows, int head_dim,
                   bool unit8) {
  auto fn = encode_tiled_fn();
  if (!fn) return false;
  CUresult r;
  if (unit8) {
    // Block sizes that are odd multiples of 8: one box is 8 rows of one
    // 64-element half (2D map), so each 8-token unit of a tile is fetched
    // from its own block.
    cuuint64_t dims[2] = {(cuuint64_t)head_dim, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)head_dim * 2};
    cuuint32_t box[2] = {64, 8};
    cuuint32_t estr[2] = {1, 1};
    r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, const_cast<void *>(pool), dims, strides, box,
           estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
  }
  const int halves = head_dim / 64;
  cuuint64_t dims[3] = {64, (cuuint64_t)rows, (cuuint64_t)halves};
  cuuint64_t strides[2] = {(cuuint64_t)head_dim * 2, 128};
  cuuint32_t box[3] = {64, 16, (cuuint32_t)halves};
  cuuint32_t estr[3] = {1, 1, 1};
  r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT16, halves > 1 ? 3 : 2, const_cast<void *>(pool), dims,
         strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int cuda_status(cudaError_t e) { return e == cudaSuccess ? PKV_OK : PKV_ECUDA; }

// Process-wide decode kernel selection (pkv_set_decode_dispatch).
std::atomic<int> g_dispatch{PKV_DISPATCH_AUTO};

// Launch shape of a single-wave decode for a 16-bit call, or false when the
// persistent kernel takes the call.
//   warp mode: every context fits WAVE_WARP_TILES tiles and one partition;
//   CTA mode: S * Hkv * P CTAs (P partitions of part_tokens each, P <=
//     WAVE_MAX_PARTS) are resident at once. Under PKV_PARTITION_AUTO, P is
//     the most partitions (of at least WAVE_MIN_PART_TILES tiles) that keep
//     it so. CTAs of 8 warps when they are at most one per SM and every warp
//     gets at least two tiles, else 4;
//   split form (PKV_PARTITION_AUTO, very long contexts): `clusters` clusters
//     of WAVE_SPLIT_CLUSTER CTAs per (sequence, KV head), merged afterwards
//     through the workspace.
// Under the default selection no warp may get more than WAVE_MAX_WARP_CHAIN
// tiles.
bool plan_wave(const pkv::DecodeArgs &a, int dtype, bool auto_part, int requested_part,
               bool *warp_items, int *warps, int *parts, int *part_tokens, int *clusters) {
  *clusters = 1;
  const int mode = g_dispatch.load(std::memory_order_relaxed);
  if (mode == PKV_DISPATCH_PERSISTENT) return false;
  const long long items = (long long)a.num_seqs * a.num_kv_heads;
  const long long max_len = a.max_context_len;
  const long long max_tiles = (max_len + 15) / 16;
  const long long whole = max_tiles > 0 ? max_tiles * 16 : 16;  // one partition holds any context
  if (whole > 0x7fffffffLL) return false;
  const bool one_part = auto_part || requested_part == 0 || requested_part >= whole;
  if (mode != PKV_DISPATCH_WAVE_CTA && mode != PKV_DISPATCH_WAVE_CTA8 && one_part &&
      (max_tiles <= pkv::WAVE_WARP_TILES || mode == PKV_DISPATCH_WAVE_WARP)) {
    *warp_items = true;
    *warps = 4;
    *parts = 1;
    *part_tokens = (int)whole;
    return true;
  }
  if (mode == PKV_DISPATCH_WAVE_WARP) return false;
  // CTAs (P == 1) or clusters of P CTAs resident at once
  auto fits = [&](long long P, int nw) {
    int cap = 0;
    return pkv::decode_wave_capacity(a, dtype, false, nw, (int)P, &cap) == cudaSuccess &&
           items <= cap;
  };
  auto parts_of = [&](long long pt) { return max_len > pt ? (max_len + pt - 1) / pt : 1; };
  long long P, pt;
  if (auto_part) {
    int per_wave = 0;
    if (pkv::decode_wave_capacity(a, dtype, false, 4, 1, &per_wave) != cudaSuccess) return false;
    const long long fit = items > 0 ? per_wave / items : 0;
    const long long by_len = (max_tiles + pkv::WAVE_MIN_PART_TILES - 1) / pkv::WAVE_MIN_PART_TILES;
    long long want = fit < by_len ? fit : by_len;
    if (want > pkv::WAVE_MAX_PARTS) want = pkv::WAVE_MAX_PARTS;
    if (want < 1) want = 1;
    // Clusters of P CTAs may pack less densely than single CTAs: take fewer
    // partitions until the cluster shape holds the whole call.
    for (;; --want) {
      pt = ((max_len + want - 1) / want + 15) / 16 * 16;
      if (pt < 16) pt = 16;
      P = parts_of(pt);
      if (fits(P, 4)) break;
      if (want <= 1) return false;
    }
  } else {
    pt = requested_part > 0 ? requested_part : whole;
    P = parts_of(pt);
    if (P > pkv::WAVE_MAX_PARTS || !fits(P, 4)) return false;
  }
  if (pt > 0x7fffffffLL) return false;
  // 8-warp CTAs: at most one per SM, every warp with two tiles or more.
  int nw = 4;
  int per_wave8 = 0;  // 8-warp CTAs resident at once
  if (mode != PKV_DISPATCH_WAVE_CTA &&
      pkv::decode_wave_capacity(a, dtype, false, 8, 1, &per_wave8) == cudaSuccess) {
    auto fits8 = [&](long long P8, long long pt8) {
      return items * P8 <= per_wave8 && (mode == PKV_DISPATCH_WAVE_CTA8 || pt8 / 16 >= 16) &&
             (P8 == 1 || fits(P8, 8));
    };
    if (auto_part) {
      // As many warps or more in 8-warp CTAs: from P down to P / 2 partitions
      // (a cluster of 8-warp CTAs spans twice the SMs, so fewer fit a GPC).
      for (long long want = P; want >= 1 && 2 * want >= P; --want) {
        long long pt8 = ((max_len + want - 1) / want + 15) / 16 * 16;
        if (pt8 < 16) pt8 = 16;
        const long long P8 = parts_of(pt8);
        if (fits8(P8, pt8)) {
          nw = 8;
          P = P8;
          pt = pt8;
          break;
        }
      }
    } else if (fits8(P, pt)) {
      nw = 8;
    }
  }
  // Very long contexts on few (sequence, KV head) pairs: one cluster each
  // leaves most of the GPU idle. Several clusters of WAVE_SPLIT_CLUSTER CTAs
  // per pair then each merge their partitions into a workspace slot, and a
  // merge launch combines the slots. Taken when it shortens every warp's
  // chain of tiles by WAVE_SPLIT_MIN_GAIN tiles or more (about the cost of
  // the extra launch).
  if (auto_part && mode == PKV_DISPATCH_AUTO && a.ws_o != nullptr) {
    constexpr long long Pc = pkv::WAVE_SPLIT_CLUSTER;
    int capc = 0;
    if (pkv::decode_wave_capacity(a, dtype, false, 4, (int)Pc, &capc) == cudaSuccess &&
        items > 0) {
      long long C = capc / items;
      if (C > a.max_parts) C = a.max_parts;  // workspace slots
      for (; C >= 2; --C) {
        long long pt2 = ((max_len + C * Pc - 1) / (C * Pc) + 15) / 16 * 16;
        if (pt2 < 16 * pkv::WAVE_MIN_PART_TILES) pt2 = 16 * pkv::WAVE_MIN_PART_TILES;
        const long long C2 = (parts_of(pt2) + Pc - 1) / Pc;
        const long long chain1 = (pt / 16 + nw - 1) / nw;  // tiles per warp, one level
        const long long chain2 = (pt2 / 16 + 3) / 4;
        if (C2 >= 2 && C2 <= C && chain1 - chain2 >= pkv::WAVE_SPLIT_MIN_GAIN &&
            chain2 <= pkv::WAVE_MAX_WARP_CHAIN) {
          *warp_items = false;
          *warps = 4;
          *parts = (int)Pc;
          *part_tokens = (int)pt2;
          *clusters = (int)C2;
          return true;
        }
      }
    }
  }
  // One CTA per partition, with no balancing between them: under the default
  // selection a partition may not give a warp more than WAVE_MAX_WARP_CHAIN
  // tiles, or one long sequence among short ones would run on few CTAs while
  // the persistent kernel spreads it.
  if (mode == PKV_DISPATCH_AUTO && (pt / 16 + nw - 1) / nw > pkv::WAVE_MAX_WARP_CHAIN)
    return false;
  *warp_items = false;
  *warps = nw;
  *parts = (int)P;
  *part_tokens = (int)pt;
  return true;
}

}  // namespace

namespace pkv {

WorkspaceLayout workspace_layout(long long S, long long Hq, long long D, long long max_parts) {
  WorkspaceLayout w{};
  size_t off = 0;
  w.sched_off = off;
  off += 256;
  w.work_off = off;
  off += round_up((size_t)(S * max_parts) * sizeof(uint2), 256);
  w.grp_off = off;  // grp[S], then grp_tiles[S]
  off += round_up((size_t)(2 * S) * sizeof(int32_t), 256);
  if (max_parts > 1) {
    const long long chunks = (max_parts + pkv::MERGE_CHUNK - 1) / pkv::MERGE_CHUNK;
    w.cnt_off = off;  // Hq >= Hkv bounds the (sequence, KV head) counters
    off += round_up((size_t)(S * Hq * chunks) * sizeof(int32_t), 256);
    w.cnt2_off = off;
    off += round_up((size_t)(S * Hq) * sizeof(int32_t), 256);
    w.o_off = off;
    off += round_up((size_t)(S * Hq * max_parts * D) * sizeof(float), 256);
    w.lse_off = off;
    off += round_up((size_t)(S * Hq * max_parts) * sizeof(float), 256);
    if (chunks > 1) {
      w.o2_off = off;
      off += round_up((size_t)(S * Hq * chunks * D) * sizeof(float), 256);
      w.lse2_off = off;
      off += round_up((size_t)(S * Hq * chunks) * sizeof(float), 256);
    }
  }
  w.tail_slots = S * Hq * max_parts < pkv::TAIL_MAX_PIECES ? S * Hq * max_parts
                                                           : pkv::TAIL_MAX_PIECES;
  w.tcnt_off = off;
  off += round_up((size_t)w.tail_slots * sizeof(int32_t), 256);
  w.to_off = off;
  off += round_up((size_t)(w.tail_slots * pkv::TAIL_COLS * D) * sizeof(float), 256);
  w.tlse_off = off;
  off += round_up((size_t)(w.tail_slots * pkv::TAIL_COLS) * sizeof(float), 256);
  w.total = off;
  return w;
}

}  // namespace pkv

extern "C" {

const char *pkv_status_string(int status) {
  switch (status) {
    case PKV_OK:
      return "ok";
    case PKV_EINVAL:
      return "invalid argument";
    case PKV_EUNSUPPORTED:
      return "unsupported configuration";
    case PKV_ECUDA:
      return "CUDA error";
    default:
      return "unknown status";
  }
}

int pkv_resolve_partition(int num_seqs, int num_heads, int max_context_len, int partition_size) {
  if (partition_size != PKV_PARTITION_AUTO) return partition_size;
  constexpr long long kRows = 1024, kMin = 256, kMax = 2048;
  const long long rows = (long long)(num_seqs > 0 ? num_seqs : 1) * (num_heads > 0 ? num_heads : 1);
  const long long n = (kRows + rows - 1) / rows;  // partitions wanted per sequence
  const long long L = max_context_len > 0 ? max_context_len : 1;
  long long part = ((L + n - 1) / n + 15) / 16 * 16;
  if (part < kMin) part = kMin;
  if (part > kMax) part = kMax;
  return (int)part;
}

int pkv_set_decode_dispatch(int mode) {
  if (mode < PKV_DISPATCH_AUTO || mode > PKV_DISPATCH_WAVE_CTA8) return PKV_EINVAL;
  return g_dispatch.exchange(mode);
}

size_t pkv_decode_workspace_bytes(int num_seqs, int num_heads, int head_dim, int max_context_len,
                                  int partition_size) {
  partition_size = pkv_resolve_partition(num_seqs, num_heads, max_context_len, partition_size);
  if (num_seqs <= 0 || num_heads <= 0 || head_dim <= 0 || max_context_len < 0 ||
      partition_size < 0)
    return 0;
  const long long mp = parts_for(max_context_len, partition_size);
  return pkv::workspace_layout(num_seqs, num_heads, head_dim, mp).total;
}

}  // extern "C"

namespace {

// paged_attn_decode, optionally with each sequence's newest token appended in
// the same pass (k_new / v_new non-null; 16-bit only).
int decode_impl(void *out, const void *q, const void *k_pool, const void *v_pool,
                const int32_t *block_tables, const int32_t *context_lens, int num_seqs,
                int num_heads, int num_kv_heads, int head_dim, int block_size,
                int max_blocks_per_seq, int num_blocks, int max_context_len, float scale,
                int dtype, int partition_size, void *workspace, size_t workspace_bytes,
                int32_t *err, void *stream, const void *k_new, const void *v_new) {
  const bool auto_part = partition_size == PKV_PARTITION_AUTO;
  const int requested_part = partition_size;
  partition_size = pkv_resolve_partition(num_seqs, num_heads, max_context_len, partition_size);
  if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 ||
      block_size <= 0 || max_blocks_per_seq <= 0 || num_blocks <= 0 || max_context_len < 0 ||
      partition_size < 0)
    return PKV_EINVAL;
  if (dtype < PKV_F32 || dtype > PKV_BF16) return PKV_EINVAL;
  if (num_heads % num_kv_heads != 0) return PKV_EINVAL;
  if (!isfinite(scale)) return PKV_EINVAL;
  if (partition_size % 16 != 0) return PKV_EINVAL;
  if (num_seqs == 0) return PKV_OK;
  if (!out || !q || !k_pool || !v_pool || !block_tables || !context_lens) return PKV_EINVAL;
  if (head_dim != 64 && head_dim != 128) return PKV_EUNSUPPORTED;
  if (num_seqs > 65535 || num_heads > 65535) return PKV_EUNSUPPORTED;

  const uintptr_t al = dtype == PKV_F32 ? 4 : 16;
  if (!aligned(out, al) || !aligned(q, al) || !aligned(k_pool, 16) || !aligned(v_pool, 16) ||
      !aligned(block_tables, 4) || !aligned(context_lens, 4))
    return PKV_EINVAL;

  long long rows = 0;  // pool rows of the TMA view (16-bit path)
  if (dtype != PKV_F32) {
    if (block_size % 8 != 0 || block_size > 256) return PKV_EUNSUPPORTED;
    if (num_heads / num_kv_heads > 8) return PKV_EUNSUPPORTED;
    rows = (long long)num_blocks * num_kv_heads * block_size;
    if (rows > 0x7fffffffLL - 64) return PKV_EUNSUPPORTED;
  }
  const long long mp = parts_for(max_context_len, partition_size);
  if (mp > 65535) return PKV_EUNSUPPORTED;  // work-list entries pack the partition in 16 bits
  pkv::DecodeArgs a{};
  a.out = out;
  a.q = q;
  a.k_pool = k_pool;
  a.v_pool = v_pool;
  a.block_tables = block_tables;
  a.context_lens = context_lens;
  a.num_seqs = num_seqs;
  a.num_heads = num_heads;
  a.num_kv_heads = num_kv_heads;
  a.head_dim = head_dim;
  a.block_size = block_size;
  a.unit8 = block_size % 16 != 0 ? 1 : 0;
  a.max_blocks = max_blocks_per_seq;
  a.num_blocks = num_blocks;
  a.max_context_len = max_context_len;
  a.max_parts = (int)mp;
  if (partition_size > 0) {
    a.part_tokens = partition_size;
  } else {
    const long long whole = round_up((size_t)(max_context_len > 0 ? max_context_len : 1), 16);
    if (whole > 0x7fffffffLL) return PKV_EUNSUPPORTED;
    a.part_tokens = (int)whole;
  }
  a.scale_log2 = scale * 1.4426950408889634f;
  a.err = err;
  const pkv::WorkspaceLayout wl = pkv::workspace_layout(num_seqs, num_heads, head_dim, mp);
  if (!workspace || workspace_bytes < wl.total || !aligned(workspace, 256)) return PKV_EINVAL;
  char *ws = static_cast<char *>(workspace);
  a.sched = reinterpret_cast<int32_t *>(ws + wl.sched_off);
  a.work = reinterpret_cast<uint2 *>(ws + wl.work_off);
  a.grp = reinterpret_cast<int32_t *>(ws + wl.grp_off);
  a.grp_tiles = a.grp + num_seqs;
  a.tail_cnt = reinterpret_cast<int32_t *>(ws + wl.tcnt_off);
  a.tail_o = reinterpret_cast<float *>(ws + wl.to_off);
  a.tail_lse = reinterpret_cast<float *>(ws + wl.tlse_off);
  a.tail_slots = (int)wl.tail_slots;
  a.max_chunks = (int)((mp + pkv::MERGE_CHUNK - 1) / pkv::MERGE_CHUNK);
  if (mp > 1) {
    a.merge_cnt = reinterpret_cast<int32_t *>(ws + wl.cnt_off);
    a.merge_cnt2 = reinterpret_cast<int32_t *>(ws + wl.cnt2_off);
    if (a.max_chunks > 1) {
      a.ws2_o = reinterpret_cast<float *>(ws + wl.o2_off);
      a.ws2_lse = reinterpret_cast<float *>(ws + wl.lse2_off);
    }
    a.ws_o = reinterpret_cast<float *>(ws + wl.o_off);
    a.ws_lse = reinterpret_cast<float *>(ws + wl.lse_off);
  }

  a.k_new = k_new;
  a.v_new = v_new;

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (dtype == PKV_F32) {
    e = pkv::launch_decode_simt_f32(a, st);
  } else {
    CUtensorMap tmK, tmV;
    if (!make_pool_map(&tmK, k_pool, rows, head_dim, a.unit8 != 0) ||
        !make_pool_map(&tmV, v_pool, rows, head_dim, a.unit8 != 0))
      return PKV_ECUDA;
    // A call that fits one wave of CTAs: one launch, no plan, no workspace.
    bool warp_items = false;
    int wwarps = 4, wparts = 1, wtokens = 0, wclusters = 1;
    if (plan_wave(a, dtype, auto_part, requested_part, &warp_items, &wwarps, &wparts, &wtokens,
                  &wclusters)) {
      pkv::DecodeArgs b = a;  // (max_parts stays the workspace's slot stride)
      b.part_tokens = wtokens;
      b.wave_clusters = wclusters;
      e = pkv::launch_decode_wave(b, dtype, warp_items, wwarps, wparts, tmK, tmV, st);
      if (e != cudaSuccess || wclusters <= 1) return cuda_status(e);
      // combine the clusters' slots: a slot spans wparts partitions
      b.part_tokens = wtokens * wparts;
      return cuda_status(pkv::launch_merge(b, dtype, st));
    }
    // plan + decode; the partition merge is fused into the decode kernel
    return cuda_status(pkv::launch_decode_tc(a, dtype, tmK, tmV, st));
  }
  if (e != cudaSuccess) return PKV_ECUDA;
  if (mp > 1) return cuda_status(pkv::launch_merge(a, dtype, st));
  return PKV_OK;
}

}  // namespace

extern "C" {

int paged_attn_decode(void *out, const void *q, const void *k_pool, const void *v_pool,
                      const int32_t *block_tables, const int32_t *context_lens, int num_seqs,
                      int num_heads, int num_kv_heads, int head_dim, int block_size,
                      int max_blocks_per_seq, int num_blocks, int max_context_len, float scale,
                      int dtype, int partition_size, void *workspace, size_t workspace_bytes,
                      int32_t *err, void *stream) {
  return decode_impl(out, q, k_pool, v_pool, block_tables, context_lens, num_seqs, num_heads,
                     num_kv_heads, head_dim, block_size, max_blocks_per_seq, num_blocks,
                     max_context_len, scale, dtype, partition_size, workspace, workspace_bytes,
                     err, stream, nullptr, nullptr);
}

int paged_attn_decode_append(void *out, const void *q, const void *k_new, const void *v_new,
                             void *k_pool, void *v_pool, const int32_t *block_tables,
                             const int32_t *context_lens, int num_seqs, int num_heads,
                             int num_kv_heads, int head_dim, int block_size,
                             int max_blocks_per_seq, int num_blocks, int max_context_len,
                             float scale, int dtype, int partition_size, void *workspace,
                             size_t workspace_bytes, int32_t *err, void *stream) {
  if (num_seqs > 0 && (!k_new || !v_new)) return PKV_EINVAL;
  if (num_seqs > 0 && (!aligned(k_new, 16) || !aligned(v_new, 16))) return PKV_EINVAL;
  if (dtype == PKV_F32) return PKV_EUNSUPPORTED;
  return decode_impl(out, q, k_pool, v_pool, block_tables, context_lens, num_seqs, num_heads,
                     num_kv_heads, head_dim, block_size, max_blocks_per_seq, num_blocks,
                     max_context_len, scale, dtype, partition_size, workspace, workspace_bytes,
                     err, stream, k_new, v_new);
}

int kv_cache_append(void *k_pool, void *v_pool, const void *k_new, const void *v_new,
                    const int64_t *slot_mapping, int num_tokens, int num_kv_heads, int head_dim,
                    int block_size, int num_blocks, int dtype, int32_t *err, void *stream) {
  if (num_tokens < 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 || num_blocks <= 0)
    return PKV_EINVAL;
  if (dtype < PKV_F32 || dtype > PKV_BF16) return PKV_EINVAL;
  if (num_tokens == 0) return PKV_OK;
  if (!k_pool || !v_pool || !k_new || !v_new || !slot_mapping) return PKV_EINVAL;
  const int es = dtype == PKV_F32 ? 4 : 2;
  const long long row_bytes = (long long)head_dim * es;
  if (row_bytes % 16 != 0 || row_bytes > 0x7fffffffLL) return PKV_EUNSUPPORTED;
  if (!aligned(k_pool, 16) || !aligned(v_pool, 16) || !aligned(k_new, 16) || !aligned(v_new, 16) ||
      !aligned(slot_mapping, 8))
    return PKV_EINVAL;
  return cuda_status(pkv::launch_append(k_pool, v_pool, k_new, v_new, slot_mapping, num_tokens,
                                        num_kv_heads, (int)row_bytes, block_size, num_blocks, err,
                                        static_cast<cudaStream_t>(stream)));
}

int kv_block_copy(void *k_pool, void *v_pool, const int32_t *src_dst, int num_pairs,
                  int num_kv_heads, int head_dim, int block_size, int num_blocks, int dtype,
                  int32_t *err, void *stream) {
  if (num_pairs < 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 || num_blocks <= 0)
    return PKV_EINVAL;
  if (dtype < PKV_F32 || dtype > PKV_BF16) return PKV_EINVAL;
  if (num_pairs == 0) return PKV_OK;
  if (!k_pool || !v_pool || !src_dst) return PKV_EINVAL;
  const int es = dtype == PKV_F32 ? 4 : 2;
  const long long block_bytes = (long long)num_kv_heads * block_size * head_dim * es;
  if (((long long)head_dim * es) % 16 != 0) return PKV_EUNSUPPORTED;
  if (!aligned(k_pool, 16) || !aligned(v_pool, 16) || !aligned(src_dst, 4)) return PKV_EINVAL;
  return cuda_status(pkv::launch_block_copy(k_pool, v_pool, src_dst, num_pairs, block_bytes,
                                            num_blocks, err, static_cast<cudaStream_t>(stream)));
}

int pkv_check_wait_timeout(long long limit_cycles, int32_t *err, void *stream) {
  if (limit_cycles <= 0 || limit_cycles > 4000000000LL || !err || !aligned(err, 4))
    return PKV_EINVAL;
  return cuda_status(pkv::launch_wait_timeout_probe(limit_cycles, err,
                                                    static_cast<cudaStream_t>(stream)));
}

int kv_block_swap(void *dst_k, void *dst_v, const void *src_k, const void *src_v,
                  const int32_t *src_dst, int num_pairs, int num_kv_heads, int head_dim,
                  int block_size, int src_blocks, int dst_blocks, int dtype, int32_t *err,
                  void *stream) {
  if (num_pairs < 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 ||
      src_blocks <= 0 || dst_blocks <= 0)
    return PKV_EINVAL;
  if (dtype < PKV_F32 || dtype > PKV_BF16) return PKV_EINVAL;
  if (num_pairs == 0) return PKV_OK;
  if (!dst_k || !dst_v || !src_k || !src_v || !src_dst) return PKV_EINVAL;
  const int es = dtype == PKV_F32 ? 4 : 2;
  const long long block_bytes = (long long)num_kv_heads * block_size * head_dim * es;
  if (((long long)head_dim * es) % 16 != 0) return PKV_EUNSUPPORTED;
  if (!aligned(dst_k, 16) || !aligned(dst_v, 16) || !aligned(src_k, 16) || !aligned(src_v, 16) ||
      !aligned(src_dst, 4))
    return PKV_EINVAL;
  return cuda_status(pkv::launch_block_swap(dst_k, dst_v, src_k, src_v, src_dst, num_pairs,
                                            block_bytes, src_blocks, dst_blocks, err,
                                            static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
