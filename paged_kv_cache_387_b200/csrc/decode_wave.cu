// Single-wave paged decode for fp16 / bf16 on sm_100a.
//
// A small call (one sequence, a few sequences, or many sequences with contexts
// of a few blocks) does not fill the GPU for long. For it, the persistent
// decode's fixed costs decide the time: a plan launch and its completion, a
// dependent chain of work-list and block-table loads, counter round trips
// before a merge, and the descriptor hand-offs. This kernel has none of them.
// Its grid is the work itself, and it neither reads nor writes the workspace.
//
//   CTA mode. CTA (p, h, s) attends partition p of sequence s for KV head h.
//     Its four warps take tiles w, w+4, w+8, ... and combine in shared
//     memory. The P partitions of one (sequence, KV head) form one
//     thread-block cluster. Each CTA leaves its normalised partial output and
//     log2-sum-exp in its own shared memory. After a cluster barrier, rank 0
//     merges them by reading its peers' shared memory directly (distributed
//     shared memory), and a second barrier keeps the peers resident until it
//     is done.
//   Warp mode (contexts of a few tiles, one partition). Each warp attends one
//     whole (sequence, KV head) alone and writes its output. There is no
//     combine and no barrier after the start.
//
// The per-tile arithmetic is the persistent kernel's. It is the block-by-block
// online softmax over the block table of page "PagedAttention Analysis"
// (ryotta.opik.net), section 3, with the partial last block masked to the
// context length (page "PagedAttention" (newikis), section "Mathematical
// formulation"):
//   - S^T = K_tile . Q^T, with mma.sync m16n8k16 and K as the A operand from
//     the 128-byte-swizzled TMA tile;
//   - a base-2 online softmax with a lazy reference max;
//   - O^T += V^T . P^T, with V^T from ldmatrix.trans and bf16 P carried as
//     hi + lo.
// Partitions are merged as o = sum_p 2^(lse_p - M) o_p / sum_p 2^(lse_p - M).
// The fused cache-append writes each sequence's newest K/V rows into the pool
// slot of token L-1 and attends over them, as the persistent kernel does.
//
// Every copy wait is bounded. One that gives up reports PKV_DEV_WAIT_TIMEOUT.
// The warp then stops issuing and reading tiles, but it still reaches every
// barrier of its CTA and cluster, so the launch always ends.
#include <mutex>
#include <tuple>
#include <map>

#include "pkv_device.cuh"
#include "pkv_internal.h"

namespace pkv {
namespace {

constexpr int WV_TILE = 16;                // tokens per tile
// Warps per CTA, all of them consumers: 4 (two CTAs per SM at head_dim 128),
// or 8 when the call has at most one CTA per SM, so that each SM sub-partition
// still runs two warps.
constexpr int WV_HALF = WV_TILE * 128;     // one 64-element box of a tile: 16 rows x 128 B
constexpr int WV_BOX_COLS = 64;
constexpr int WV_COLS = 8;                 // score columns of the MMA: query heads of a KV head
constexpr float WV_SLACK = 8.f;            // lazy max: rescale only past 2^8 growth

template <int D, int NW>
struct WaveShape {
  static constexpr int THREADS = NW * 32;
  static constexpr int HALVES = D / WV_BOX_COLS;
  static constexpr int KT_BYTES = HALVES * WV_HALF;  // one K (or V) tile
  static constexpr int STAGE_BYTES = 2 * KT_BYTES;   // K + V
  static constexpr int NSTAGE = 3;
  static constexpr int RING_BYTES = NW * NSTAGE * STAGE_BYTES;
  // After the tiles, the ring is reused: the warps' combine rows, the CTA's
  // partial result, then the merge weights.
  static constexpr int AS = D + 4;  // padded combine row (floats)
  static constexpr int CW_FLOATS = WV_COLS * AS + 2 * WV_COLS;  // acc[8][D+4], m[8], l[8]
  static constexpr int PART_OFF = (NW * CW_FLOATS * 4 + 15) & ~15;
  static constexpr int PART_LSE_OFF = PART_OFF + WV_COLS * D * 4;
  static constexpr int WTS_OFF = PART_LSE_OFF + WV_COLS * 4;
  static constexpr int WTS_FLOATS = WV_COLS * WAVE_MAX_PARTS;  // >= the combine's [8][4] + [8]
  static constexpr int BAR_OFF = RING_BYTES;
  static constexpr int SMEM_BYTES = RING_BYTES + NW * NSTAGE * 8 + 1024;  // + alignment
  static_assert(WTS_OFF + WTS_FLOATS * 4 <= RING_BYTES, "combine areas fit in the ring");
  static_assert(WTS_FLOATS >= WV_COLS * NW + WV_COLS, "scales fit in the weights area");
  static_assert(SMEM_BYTES <= 227 * 1024, "one CTA fits an SM");
};

template <typename T, int D, bool U8, bool WARP_ITEMS, int NW>
__global__ void __launch_bounds__(NW * 32, 8 / NW)
    decode_wave_kernel(const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const DecodeArgs a) {
  using Shape = WaveShape<D, NW>;
  constexpr int WV_WARPS = NW;
  constexpr int WV_THREADS = Shape::THREADS;
  constexpr int NSTAGE = Shape::NSTAGE;
  constexpr int AS = Shape::AS;
  constexpr int CH = D / 8;  // 16-byte chunks per K or V row
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_addr(smem_raw);
  const uint32_t smem0 = (raw_addr + 1023u) & ~1023u;  // 128B swizzle wants 1024B alignment
  uint8_t *const sm = smem_raw + (smem0 - raw_addr);

  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int Hq = a.num_heads;
  const int Hkv = a.num_kv_heads;
  const int G = Hq / Hkv;
  const int B = a.block_size;
  const uint32_t bars = smem0 + Shape::BAR_OFF;
  const uint32_t ring = smem0 + warp * NSTAGE * Shape::STAGE_BYTES;
  auto tile_full = [&](int st) { return bars + 8 * (warp * NSTAGE + st); };

  if (threadIdx.x == 0) {
    for (int i = 0; i < WV_WARPS * NSTAGE; ++i) mbar_init(bars + 8 * i, 1);
    fence_mbar_init();
    prefetch_tensormap(&tmK);
    prefetch_tensormap(&tmV);
  }
  __syncthreads();
  // The next launch in the stream may start its set-up; it waits for this
  // grid to complete before it touches memory. This grid waits likewise for
  // the one before it (which may write the context lengths or the pool).
  pdl_launch_dependents();
  pdl_wait();
  // A call that starts after some wait already gave up does no work: no
  // output, no append (the caller resets the error word first). The decision
  // is taken once per CTA, so that its barriers stay uniform.
  const bool stale = __syncthreads_or(threadIdx.x == 0 && a.err != nullptr &&
                                      *reinterpret_cast<volatile const int32_t *>(a.err) ==
                                          PKV_DEV_WAIT_TIMEOUT) != 0;

  // ---- the work of this warp ----
  int s, h, p;
  bool active;
  if constexpr (WARP_ITEMS) {
    const long long item = (long long)blockIdx.x * WV_WARPS + warp;
    active = !stale && item < (long long)a.num_seqs * Hkv;
    s = active ? (int)(item / Hkv) : 0;
    h = active ? (int)(item - (long long)s * Hkv) : 0;
    p = 0;
  } else {
    // blockIdx.z = s * C + c: cluster c of sequence s's KV head h holds
    // partitions c * P .. c * P + P - 1, one per CTA (rank blockIdx.x).
    const int C = max(1, a.wave_clusters);
    h = blockIdx.y;
    s = blockIdx.z / C;
    p = (blockIdx.z - s * C) * gridDim.x + blockIdx.x;
    active = !stale;
  }
  const int raw_len = active ? __ldg(a.context_lens + s) : 0;
  const int L = effective_len(raw_len, a.max_context_len, a.max_blocks, B,
                              lane == 0 && h == 0 && p == 0 ? a.err : nullptr);
  const int tiles = (L + WV_TILE - 1) / WV_TILE;
  const int ptiles = a.part_tokens / WV_TILE;
  const int nparts = tiles > ptiles ? (tiles + ptiles - 1) / ptiles : 1;
  const int tile0 = p * ptiles;
  const int n_tiles = min(ptiles, max(0, tiles - tile0));  // this CTA's (or warp's) tiles
  const int nt_w = WARP_ITEMS ? n_tiles
                              : (warp < n_tiles ? (n_tiles - warp + WV_WARPS - 1) / WV_WARPS : 0);
  auto tile_of = [&](int j) { return WARP_ITEMS ? tile0 + j : tile0 + warp + j * WV_WARPS; };

  // Physical block ids of this warp's tiles ids_base .. ids_base + 31: lane k
  // holds tile ids_base + k's (and with 8-token units, its second unit's).
  const int32_t *const bt = a.block_tables + (size_t)s * a.max_blocks;
  int id0 = -1, id1 = -1, ids_base = 0;
  auto load_ids = [&](int base) {
    const int j = base + lane;
    id0 = -1;
    id1 = -1;
    if (j < nt_w) {
      const int tok0 = tile_of(j) * WV_TILE;
      id0 = __ldg(bt + tok0 / B);
      if (U8 && tok0 + WV_TILE / 2 < L) id1 = __ldg(bt + (tok0 + WV_TILE / 2) / B);
    }
  };
  load_ids(0);

  // Fused append: the warp whose tile holds token L-1 takes that token's K
  // (lanes < CH) or V (lanes CH .. 2CH-1) chunk from k_new / v_new now, and
  // its pool block.
  int j_new = -1;
  if (a.k_new != nullptr && L > 0) {
    const int rel = (L - 1) / WV_TILE - tile0;
    if (rel >= 0 && rel < n_tiles) {
      if (WARP_ITEMS)
        j_new = rel;
      else if (rel % WV_WARPS == warp)
        j_new = rel / WV_WARPS;
    }
  }
  const int e_ch = lane % CH, kv_ch = lane / CH;
  uint4 newest = make_uint4(0u, 0u, 0u, 0u);
  int new_blk = 0;
  if (j_new >= 0) {
    if (lane < 2 * CH) {
      const T *src = static_cast<const T *>(kv_ch ? a.v_new : a.k_new) +
                     ((size_t)s * Hkv + h) * D + e_ch * 8;
      newest = __ldg(reinterpret_cast<const uint4 *>(src));
    }
    new_blk = __ldg(bt + (L - 1) / B);
  }

  // Q^T as the B operand: lane (g, c) holds head g's elements
  // 8*Lc .. 8*Lc+7 for logical chunk Lc(c, j) = (j/2)*8 + 2c + (j%2).
  const int g = lane >> 2;  // mma group id (row of A / column of B)
  const int c = lane & 3;   // thread in group
  uint4 qf[D / 32];
  {
    const bool live = g < G && nt_w > 0;
    const T *qrow = static_cast<const T *>(a.q) + ((size_t)s * Hq + h * G + min(g, G - 1)) * D;
#pragma unroll
    for (int j = 0; j < D / 32; ++j) {
      const int Lc = (j >> 1) * 8 + 2 * c + (j & 1);
      qf[j] = live ? __ldg(reinterpret_cast<const uint4 *>(qrow + Lc * 8))
                   : make_uint4(0u, 0u, 0u, 0u);
    }
  }

  // ---- issue side: lane 0 fills the warp's ring with TMA ----
  const int total_rows = a.num_blocks * Hkv * B;
  uint32_t issued = 0, done = 0;
  uint32_t bad_mask = 0;  // bit st: the tile in stage st had an invalid block id
  auto issue = [&]() {
    const int j = (int)issued;
    if (j - ids_base >= 32) {
      ids_base += 32;
      load_ids(ids_base);
    }
    const int k = j - ids_base;
    const int p0 = __shfl_sync(FULL_MASK, id0, k);
    const int p1 = __shfl_sync(FULL_MASK, id1, k);
    const int tok0 = tile_of(j) * WV_TILE;
    // Pool row of each unit of the tile. total_rows is wholly out of bounds
    // (TMA fills zeros): it stands for an invalid block id, which is reported,
    // and for a second unit past the context, whose table entry is not read.
    bool bad = p0 < 0 || p0 >= a.num_blocks;
    const int y0 = bad ? total_rows : (p0 * Hkv + h) * B + (tok0 % B);
    int y1 = total_rows;
    if (U8 && tok0 + WV_TILE / 2 < L) {
      const bool bad1 = p1 < 0 || p1 >= a.num_blocks;
      bad = bad || bad1;
      if (!bad1) y1 = (p1 * Hkv + h) * B + ((tok0 + WV_TILE / 2) % B);
    }
    const int st = issued % NSTAGE;
    bad_mask = bad ? (bad_mask | (1u << st)) : (bad_mask & ~(1u << st));
    if (lane == 0) {
      if (bad) report(a.err, PKV_DEV_BAD_BLOCK);
      const uint32_t bar = tile_full(st);
      const uint32_t kdst = ring + st * Shape::STAGE_BYTES;
      const uint32_t vdst = kdst + Shape::KT_BYTES;
      mbar_arrive_expect_tx(bar, Shape::STAGE_BYTES);
      if constexpr (U8) {
        // two 8-row boxes per 64-element half (2D map): rows 0-7 and 8-15
#pragma unroll
        for (int hh = 0; hh < Shape::HALVES; ++hh) {
          const uint32_t o = hh * WV_HALF;
          tma_load_2d(kdst + o, &tmK, hh * WV_BOX_COLS, y0, bar);
          tma_load_2d(kdst + o + WV_HALF / 2, &tmK, hh * WV_BOX_COLS, y1, bar);
          tma_load_2d(vdst + o, &tmV, hh * WV_BOX_COLS, y0, bar);
          tma_load_2d(vdst + o + WV_HALF / 2, &tmV, hh * WV_BOX_COLS, y1, bar);
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
  };
  while ((int)issued < min(nt_w, NSTAGE)) issue();

  // ---- consume side ----
  float acc[D / 16][4];
#pragma unroll
  for (int mt = 0; mt < D / 16; ++mt) acc[mt][0] = acc[mt][1] = acc[mt][2] = acc[mt][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY;  // reference max of heads 2c, 2c+1 (base-2 units)
  float l0 = 0.f, l1 = 0.f;              // this lane's share of the running sums
  const float sl2 = a.scale_log2;
  const bool col0_live = 2 * c < G, col1_live = 2 * c + 1 < G;
  const int mi = lane >> 3;                      // ldmatrix: lane feeds row (lane & 7)
  const int vr = (lane & 7) + ((mi >> 1) << 3);  //   of matrix mi; token row in the tile

  for (int j = 0; j < nt_w; ++j) {
    const int st = done % NSTAGE;
    if (!__all_sync(FULL_MASK, mbar_wait_bounded(tile_full(st), (done / NSTAGE) & 1))) {
      if (lane == 0) report(a.err, PKV_DEV_WAIT_TIMEOUT);
      break;
    }
    const uint32_t ks = ring + st * Shape::STAGE_BYTES;
    const uint32_t vs = ks + Shape::KT_BYTES;
    const int tok0 = tile_of(j) * WV_TILE;
    const int valid = min(WV_TILE, L - tok0);
    const bool bad = (bad_mask >> st) & 1u;

    if (j == j_new && !bad) {
      // Fused append: this tile holds token L-1. Its K and V rows come from
      // the new rows (whatever the pool slot held), and the same rows are
      // written to the pool slot: that is the cache-append.
      const int r = L - 1 - tok0;
      if (lane < 2 * CH) {
        const uint32_t tb = kv_ch ? vs : ks;
        sts128(tb + (e_ch >> 3) * WV_HALF + r * 128 + (((e_ch & 7) ^ (r & 7)) << 4), newest);
        T *pool = static_cast<T *>(const_cast<void *>(kv_ch ? a.v_pool : a.k_pool));
        *reinterpret_cast<uint4 *>(pool + (((size_t)new_blk * Hkv + h) * B + (L - 1) % B) * D +
                                   e_ch * 8) = newest;
      }
      fence_proxy_async_smem();  // these writes precede the stage's next TMA fill
      __syncwarp();
    }
    if (valid < WV_TILE && !bad) {
      // Tokens past the context length: their V rows may hold anything (NaN
      // included); zero them so P*V stays finite.
      const int nchunks = (WV_TILE - valid) * 8 * Shape::HALVES;
      for (int e = lane; e < nchunks; e += 32) {
        const int r = valid + e / (8 * Shape::HALVES);
        const int rem = e % (8 * Shape::HALVES);
        sts128_zero(vs + (rem >> 3) * WV_HALF + r * 128 + (rem & 7) * 16);
      }
      fence_proxy_async_smem();
      __syncwarp();
    }

    // ---- scores: S^T = K . Q^T (two independent accumulation chains) ----
    float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int jj = 0; jj < D / 32; ++jj) {
      const int Lc = (jj >> 1) * 8 + 2 * c + (jj & 1);
      const uint32_t rowg = ks + (Lc >> 3) * WV_HALF + g * 128 + (((Lc & 7) ^ g) << 4);
      const uint4 ka = lds128(rowg);            // token g
      const uint4 kb = lds128(rowg + 8 * 128);  // token g + 8 (same swizzle phase)
      mma16816<T>(sa, ka.x, kb.x, ka.y, kb.y, qf[jj].x, qf[jj].y);
      mma16816<T>(sb, ka.z, kb.z, ka.w, kb.w, qf[jj].z, qf[jj].w);
    }

    // ---- online softmax (heads 2c, 2c+1; tokens g, g+8) ----
    const bool ok0 = !bad && g < valid;
    const bool ok1 = !bad && g + 8 < valid;
    const float x0 = ok0 && col0_live ? (sa[0] + sb[0]) * sl2 : -INFINITY;
    const float x1 = ok0 && col1_live ? (sa[1] + sb[1]) * sl2 : -INFINITY;
    const float x2 = ok1 && col0_live ? (sa[2] + sb[2]) * sl2 : -INFINITY;
    const float x3 = ok1 && col1_live ? (sa[3] + sb[3]) * sl2 : -INFINITY;
    float mx0 = fmaxf(x0, x2), mx1 = fmaxf(x1, x3);
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      mx0 = fmaxf(mx0, __shfl_xor_sync(FULL_MASK, mx0, off));
      mx1 = fmaxf(mx1, __shfl_xor_sync(FULL_MASK, mx1, off));
    }
    const bool up0 = mx0 > m0 + WV_SLACK, up1 = mx1 > m1 + WV_SLACK;
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

    // P^T as the B operand (bf16: hi + lo parts, two MMAs; fp16: one).
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
      const uint32_t addr = vrow + (chunk >> 3) * WV_HALF + (((chunk & 7) ^ (vr & 7)) << 4);
      uint32_t r0, r1, r2, r3;
      ldsm_x4_trans(addr, r0, r1, r2, r3);
      mma16816<T>(acc[mt], r0, r1, r2, r3, pb0, pb1);
      if constexpr (kSplitP) mma16816<T>(acc[mt], r0, r1, r2, r3, pl0, pl1);
    }
    __syncwarp();  // every lane is done with this stage before it is refilled
    ++done;
    if ((int)issued < nt_w) issue();
  }
  // After a wait gave up, copies this warp issued may still be landing in its
  // ring: wait for them (bounded) before the ring is reused or released.
  for (; done != issued; ++done)
    if (!__all_sync(FULL_MASK, mbar_wait_bounded(tile_full(done % NSTAGE), (done / NSTAGE) & 1)))
      break;

  // Full per-warp sums: add the 8 lanes that share a head pair.
#pragma unroll
  for (int off = 4; off < 32; off <<= 1) {
    l0 += __shfl_xor_sync(FULL_MASK, l0, off);
    l1 += __shfl_xor_sync(FULL_MASK, l1, off);
  }

  if constexpr (WARP_ITEMS) {
    // One warp, one (sequence, KV head), one partition: normalise and store.
    if (!active) return;
    const float i0 = l0 > 0.f ? 1.f / l0 : 0.f, i1 = l1 > 0.f ? 1.f / l1 : 0.f;
    T *const out = static_cast<T *>(a.out) + ((size_t)s * Hq + h * G) * D;
#pragma unroll
    for (int mt = 0; mt < D / 16; ++mt) {
      if (col0_live) {
        out[(2 * c) * D + 16 * mt + g] = from_float<T>(acc[mt][0] * i0);
        out[(2 * c) * D + 16 * mt + g + 8] = from_float<T>(acc[mt][2] * i0);
      }
      if (col1_live) {
        out[(2 * c + 1) * D + 16 * mt + g] = from_float<T>(acc[mt][1] * i1);
        out[(2 * c + 1) * D + 16 * mt + g + 8] = from_float<T>(acc[mt][3] * i1);
      }
    }
  } else {
    // ---- combine the four warps (the ring is free now) ----
    __syncthreads();
    float *const areas = reinterpret_cast<float *>(sm);
    float *const cw = areas + warp * Shape::CW_FLOATS;
#pragma unroll
    for (int mt = 0; mt < D / 16; ++mt) {
      if (col0_live) {
        cw[(2 * c) * AS + 16 * mt + g] = acc[mt][0];
        cw[(2 * c) * AS + 16 * mt + g + 8] = acc[mt][2];
      }
      if (col1_live) {
        cw[(2 * c + 1) * AS + 16 * mt + g] = acc[mt][1];
        cw[(2 * c + 1) * AS + 16 * mt + g + 8] = acc[mt][3];
      }
    }
    if (g == 0) {
      if (col0_live) {
        cw[WV_COLS * AS + 2 * c] = m0;
        cw[WV_COLS * AS + WV_COLS + 2 * c] = l0;
      }
      if (col1_live) {
        cw[WV_COLS * AS + 2 * c + 1] = m1;
        cw[WV_COLS * AS + WV_COLS + 2 * c + 1] = l1;
      }
    }
    __syncthreads();
    float *const sc = reinterpret_cast<float *>(sm + Shape::WTS_OFF);  // [8][4] warp weights
    float *const part_o = reinterpret_cast<float *>(sm + Shape::PART_OFF);
    float *const part_lse = reinterpret_cast<float *>(sm + Shape::PART_LSE_OFF);
    if (threadIdx.x < G) {
      // per column: warp weights 2^(m_w - M) / sum, and the log2-sum-exp
      const int n = threadIdx.x;
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < WV_WARPS; ++w)
        M = fmaxf(M, areas[w * Shape::CW_FLOATS + WV_COLS * AS + n]);
      float f[WV_WARPS], den = 0.f;
#pragma unroll
      for (int w = 0; w < WV_WARPS; ++w) {
        const float mw = areas[w * Shape::CW_FLOATS + WV_COLS * AS + n];
        f[w] = (M == -INFINITY || mw == -INFINITY) ? 0.f : ex2_approx(mw - M);
        den += f[w] * areas[w * Shape::CW_FLOATS + WV_COLS * AS + WV_COLS + n];
      }
      const float inv = den > 0.f ? 1.f / den : 0.f;
#pragma unroll
      for (int w = 0; w < WV_WARPS; ++w) sc[n * WV_WARPS + w] = f[w] * inv;
      part_lse[n] = den > 0.f ? M + lg2_approx(den) : -INFINITY;
    }
    __syncthreads();
    const bool direct = nparts == 1;
    if (active && (!direct || p == 0)) {  // (uniform over the CTA)
      T *const out = static_cast<T *>(a.out) + ((size_t)s * Hq + h * G) * D;
      for (int idx = threadIdx.x; idx < G * D; idx += WV_THREADS) {
        const int n = idx / D;
        const int dd = idx - n * D;
        float o = 0.f;
#pragma unroll
        for (int w = 0; w < WV_WARPS; ++w)
          o += sc[n * WV_WARPS + w] * areas[w * Shape::CW_FLOATS + n * AS + dd];
        if (direct)
          out[idx] = from_float<T>(o);
        else
          part_o[idx] = o;
      }
    }

    if (gridDim.x > 1) {  // a cluster of the P partitions (uniform over the cluster)
      cluster_sync_all();  // every partition's result is in its CTA's shared memory
      // This cluster's partitions q0 .. q0 + cnt - 1 of the sequence's nparts.
      // With at most one cluster's worth, rank 0 writes the output; otherwise
      // it writes the cluster's result (normalised o, log2-sum-exp) to
      // workspace slot q0 / P, for the merge launch that follows.
      const int P = gridDim.x;
      const int q0 = p - blockIdx.x;
      const int cnt = min(P, nparts - q0);
      const bool to_out = nparts <= P;
      if (active && blockIdx.x == 0 && nparts > 1 && cnt >= 1) {  // (uniform over the CTA)
        float *const wts = sc;  // [8][WAVE_MAX_PARTS] partition weights (scales are done)
        if (threadIdx.x < G) {
          const int n = threadIdx.x;
          const uint32_t lse_addr = smem_addr(part_lse + n);
          float lq[WAVE_MAX_PARTS];
          float M = -INFINITY;
#pragma unroll
          for (int q = 0; q < WAVE_MAX_PARTS; ++q) {
            lq[q] = q < cnt ? ld_cluster_f32(cluster_map(lse_addr, q)) : -INFINITY;
            M = fmaxf(M, lq[q]);
          }
          float W = 0.f;
#pragma unroll
          for (int q = 0; q < WAVE_MAX_PARTS; ++q) {
            lq[q] = (M == -INFINITY || lq[q] == -INFINITY) ? 0.f : ex2_approx(lq[q] - M);
            W += lq[q];
          }
          const float inv = W > 0.f ? 1.f / W : 0.f;
#pragma unroll
          for (int q = 0; q < WAVE_MAX_PARTS; ++q) wts[n * WAVE_MAX_PARTS + q] = lq[q] * inv;
          if (!to_out)
            a.ws_lse[((size_t)s * Hq + h * G + n) * a.max_parts + q0 / P] =
                W > 0.f ? M + lg2_approx(W) : -INFINITY;
        }
        __syncthreads();
        T *const out = static_cast<T *>(a.out) + ((size_t)s * Hq + h * G) * D;
        const uint32_t po = smem_addr(part_o);
        for (int idx = threadIdx.x * 4; idx < G * D; idx += WV_THREADS * 4) {
          const int n = idx / D;
          float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
          for (int q = 0; q < cnt; ++q) {
            const float w = wts[n * WAVE_MAX_PARTS + q];
            const float4 v = ld_cluster_f32x4(cluster_map(po + idx * 4, q));
            o.x += w * v.x;
            o.y += w * v.y;
            o.z += w * v.z;
            o.w += w * v.w;
          }
          if (to_out) {
            uint2 packed;
            packed.x = pack2<T>(o.x, o.y);
            packed.y = pack2<T>(o.z, o.w);
            *reinterpret_cast<uint2 *>(out + idx) = packed;
          } else {
            const size_t row = (size_t)s * Hq + h * G + n;
            *reinterpret_cast<float4 *>(a.ws_o + (row * a.max_parts + q0 / P) * D + (idx - n * D)) =
                o;
          }
        }
      }
      cluster_sync_all();  // rank 0 has finished reading its peers' shared memory
    }
  }
}

// Per-SM residency of a kernel instance, and the most clusters of P CTAs
// that can be resident at once, both cached per device.
std::mutex g_wave_mu;
std::map<std::tuple<int, const void *, int>, int> g_wave_cache;

template <typename Kern>
cudaError_t cached_capacity(Kern kern, int smem, int threads, int cluster, int dev, int *out) {
  const auto key = std::make_tuple(dev, reinterpret_cast<const void *>(kern), cluster);
  {
    std::lock_guard<std::mutex> lock(g_wave_mu);
    auto it = g_wave_cache.find(key);
    if (it != g_wave_cache.end()) {
      *out = it->second;
      return cudaSuccess;
    }
  }
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  int v = 0;
  if (cluster <= 1) {
    int per_sm = 0, sms = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, smem);
    if (e != cudaSuccess) return e;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    v = per_sm * sms;  // CTAs of one wave
  } else {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)cluster, 1, 1);
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)cluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaOccupancyMaxActiveClusters(&v, kern, &cfg);
    if (e != cudaSuccess) {
      cudaGetLastError();  // an unsupported cluster shape: not eligible
      v = 0;
    }
  }
  std::lock_guard<std::mutex> lock(g_wave_mu);
  g_wave_cache[key] = v;
  *out = v;
  return cudaSuccess;
}

template <typename T, int D, bool U8, bool WI, int NW>
cudaError_t wave_capacity_t(int cluster, int *out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  using Shape = WaveShape<D, NW>;
  return cached_capacity(decode_wave_kernel<T, D, U8, WI, NW>, Shape::SMEM_BYTES, Shape::THREADS,
                         cluster, dev, out);
}

template <typename T, int D, bool U8, bool WI, int NW>
cudaError_t launch_wave_t(const DecodeArgs &a, int parts, const CUtensorMap &tmK,
                          const CUtensorMap &tmV, cudaStream_t stream) {
  using Shape = WaveShape<D, NW>;
  auto kern = decode_wave_kernel<T, D, U8, WI, NW>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       Shape::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  if (!WI && parts > 8) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  if (WI) {
    const long long items = (long long)a.num_seqs * a.num_kv_heads;
    cfg.gridDim = dim3((unsigned)((items + NW - 1) / NW));
  } else {
    cfg.gridDim = dim3((unsigned)parts, (unsigned)a.num_kv_heads,
                       (unsigned)(a.num_seqs * max(1, a.wave_clusters)));
  }
  cfg.blockDim = dim3(Shape::THREADS);
  cfg.dynamicSmemBytes = Shape::SMEM_BYTES;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  int n = 1;
  if (!WI && parts > 1) {
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = (unsigned)parts;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    n = 2;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kern, tmK, tmV, a);
}

template <typename T, bool U8, bool WI, int NW>
cudaError_t wave_dispatch_d(bool launch, const DecodeArgs &a, int parts, const CUtensorMap *tmK,
                            const CUtensorMap *tmV, cudaStream_t stream, int *cap) {
  if (a.head_dim == 64)
    return launch ? launch_wave_t<T, 64, U8, WI, NW>(a, parts, *tmK, *tmV, stream)
                  : wave_capacity_t<T, 64, U8, WI, NW>(WI ? 1 : parts, cap);
  return launch ? launch_wave_t<T, 128, U8, WI, NW>(a, parts, *tmK, *tmV, stream)
                : wave_capacity_t<T, 128, U8, WI, NW>(WI ? 1 : parts, cap);
}

// Warp form: 4 warps per CTA. CTA form: 4 or 8 warps.
template <typename T, bool U8>
cudaError_t wave_dispatch_u(bool launch, const DecodeArgs &a, bool warp_items, int warps,
                            int parts, const CUtensorMap *tmK, const CUtensorMap *tmV,
                            cudaStream_t stream, int *cap) {
  if (warp_items)
    return wave_dispatch_d<T, U8, true, 4>(launch, a, parts, tmK, tmV, stream, cap);
  if (warps == 8)
    return wave_dispatch_d<T, U8, false, 8>(launch, a, parts, tmK, tmV, stream, cap);
  return wave_dispatch_d<T, U8, false, 4>(launch, a, parts, tmK, tmV, stream, cap);
}

template <typename T>
cudaError_t wave_dispatch(bool launch, const DecodeArgs &a, bool warp_items, int warps, int parts,
                          const CUtensorMap *tmK, const CUtensorMap *tmV, cudaStream_t stream,
                          int *cap) {
  return a.unit8 ? wave_dispatch_u<T, true>(launch, a, warp_items, warps, parts, tmK, tmV, stream,
                                            cap)
                 : wave_dispatch_u<T, false>(launch, a, warp_items, warps, parts, tmK, tmV,
                                             stream, cap);
}

}  // namespace

cudaError_t decode_wave_capacity(const DecodeArgs &a, int dtype, bool warp_items, int warps,
                                 int parts, int *cap) {
  *cap = 0;
  return dtype == PKV_BF16
             ? wave_dispatch<__nv_bfloat16>(false, a, warp_items, warps, parts, nullptr, nullptr,
                                            nullptr, cap)
             : wave_dispatch<__half>(false, a, warp_items, warps, parts, nullptr, nullptr,
                                     nullptr, cap);
}

cudaError_t launch_decode_wave(const DecodeArgs &a, int dtype, bool warp_items, int warps,
                               int parts, const CUtensorMap &tmK, const CUtensorMap &tmV,
                               cudaStream_t stream) {
  return dtype == PKV_BF16
             ? wave_dispatch<__nv_bfloat16>(true, a, warp_items, warps, parts, &tmK, &tmV, stream,
                                            nullptr)
             : wave_dispatch<__half>(true, a, warp_items, warps, parts, &tmK, &tmV, stream,
                                     nullptr);
}

}  // namespace pkv
