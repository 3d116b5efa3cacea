// Paged decode attention for fp16 / bf16 on sm_100a.
//
// One CTA attends one (sequence, KV head, partition). It serves all
// G = Hq/Hkv query heads of the KV head's group at once, so each K/V byte
// is read from HBM once per group.
//
// The block-by-block online softmax is the walk over the block table in page
// "PagedAttention Analysis" (ryotta.opik.net), section 3: look up each logical
// block's physical block, score it, update a running max / denominator /
// output. The partial last block is masked to the context length, which is
// the causal sum of page "PagedAttention" (newikis), section "Mathematical
// formulation".
//
// Data movement
//   The unit of work is a 16-token tile of one KV head: 16 rows of head_dim
//   elements, a slice of one physical block (block_size is a multiple of 16).
//   Each warp owns a 3-stage ring in shared memory. Lane 0 fetches a tile's K
//   and V with 2D TMA loads of 64-element-wide boxes under the 128-byte
//   swizzle and completes them on an mbarrier. A warp walks tiles w, w+4,
//   w+8, ... of the partition. No load uses cluster multicast.
//
// Math (per tile, per warp), fp32 accumulation:
//   S^T[16 tok][8 heads] = K_tile[16][D] . Q^T[D][8]  mma.sync m16n8k16. K is
//     the A operand, read straight from the swizzled tile. The D axis is
//     visited in a lane-dependent order that Q's fragments follow too, which
//     keeps every shared load a conflict-free 16-byte access. Q (G <= 8 heads,
//     zero-padded to 8) stays in registers for the whole tile loop.
//   online softmax in base 2 on the accumulator fragment. Masked tokens get
//     -inf, and the V rows of masked tokens are zeroed in shared memory before
//     they reach the tensor core.
//   O^T[D][8] += V^T[D][16] . P^T[16][8]  V^T via ldmatrix.trans; P^T from the
//     score fragment via movmatrix.trans (P rounded to the input type).
// At the end the four warps' (max, sum, output) are combined in shared
// memory. The result is written to `out` when the sequence has one partition,
// and otherwise to the workspace as (normalised o_p, log2-sum-exp) for the
// merge kernel.
#include "pkv_device.cuh"
#include "pkv_internal.h"

namespace pkv {
namespace {

constexpr int TILE = 16;                   // tokens per tile (mma M for QK, K for PV)
constexpr int NWARPS = 4;                  // warps per CTA
constexpr int NSTAGE = 3;                  // ring depth per warp
constexpr int BOX_COLS = 64;               // elements per TMA box row (128 bytes)
constexpr int HALF_BYTES = TILE * 128;     // one box: 16 rows x 128 bytes

template <int D>
struct TcShape {
  static constexpr int HALVES = D / BOX_COLS;
  static constexpr int KT_BYTES = HALVES * HALF_BYTES;     // one K (or V) tile
  static constexpr int STAGE_BYTES = 2 * KT_BYTES;         // K + V
  static constexpr int RING_BYTES = NWARPS * NSTAGE * STAGE_BYTES;
  static constexpr int BAR_BYTES = NWARPS * NSTAGE * 8;
  static constexpr int SMEM_BYTES = RING_BYTES + BAR_BYTES + 1024;  // + alignment slack
  static constexpr int ACC_STRIDE = D + 4;  // padded row of the combine area (floats)
  static_assert(8 * ACC_STRIDE * 4 + 64 <= NSTAGE * STAGE_BYTES, "combine area must fit");
};

template <typename T, int D>
__global__ void __launch_bounds__(NWARPS * 32)
    decode_tc_kernel(const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const DecodeArgs a) {
  using Shape = TcShape<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_addr(smem_raw);
  const uint32_t smem0 = (raw_addr + 1023u) & ~1023u;  // 128B swizzle wants 1024B alignment
  uint8_t *const smem_gen = smem_raw + (smem0 - raw_addr);

  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int g = lane >> 2;  // mma group id (row of A / column of B)
  const int c = lane & 3;   // thread in group
  const int p = blockIdx.x;
  const int h = blockIdx.y;
  const int s = blockIdx.z;
  const int Hq = a.num_heads;
  const int G = Hq / a.num_kv_heads;
  const int B = a.block_size;

  const int L = effective_len(a.context_lens[s], a.max_context_len, a.max_blocks, B,
                              threadIdx.x == 0 ? a.err : nullptr);
  T *const out = static_cast<T *>(a.out);
  if (L <= 0) {
    if (p == 0)
      for (int idx = threadIdx.x; idx < G * D; idx += NWARPS * 32)
        out[((size_t)s * Hq + h * G) * D + idx] = from_float<T>(0.f);
    return;
  }
  const int t_begin = p * a.part_tokens;
  if (t_begin >= L) return;
  const int t_end = min(L, t_begin + a.part_tokens);
  const int n_tiles = (t_end - t_begin + TILE - 1) / TILE;
  const int nparts = (L + a.part_tokens - 1) / a.part_tokens;
  const int nt_w = warp < n_tiles ? (n_tiles - warp + NWARPS - 1) / NWARPS : 0;

  const uint32_t ring = smem0 + warp * NSTAGE * Shape::STAGE_BYTES;
  const uint32_t bar0 = smem0 + Shape::RING_BYTES + warp * NSTAGE * 8;
  if (lane == 0) {
    for (int st = 0; st < NSTAGE; ++st) mbar_init(bar0 + 8 * st, 1);
    fence_mbar_init();
  }
  if (threadIdx.x == 0) {
    prefetch_tensormap(&tmK);
    prefetch_tensormap(&tmV);
  }
  __syncwarp();

  // Q^T as the B operand: lane (g, c) holds head g's elements
  // 8*Lc .. 8*Lc+7 for logical chunk Lc(c, j) = (j/2)*8 + 2c + (j%2).
  uint4 qf[D / 32];
  {
    const bool head_ok = g < G;
    const T *qrow = static_cast<const T *>(a.q) + ((size_t)s * Hq + h * G + (head_ok ? g : 0)) * D;
#pragma unroll
    for (int j = 0; j < D / 32; ++j) {
      const int Lc = (j >> 1) * 8 + 2 * c + (j & 1);
      qf[j] = head_ok ? *reinterpret_cast<const uint4 *>(qrow + Lc * 8) : make_uint4(0, 0, 0, 0);
    }
  }

  // Physical block ids of this warp's tiles, 32 at a time (lane j <-> tile win_base + j).
  const int32_t *bt = a.block_tables + (size_t)s * a.max_blocks;
  auto tile_tok0 = [&](int i) { return t_begin + (warp + i * NWARPS) * TILE; };
  int win_base = 0;
  int win_id = lane < nt_w ? bt[tile_tok0(lane) / B] : -1;
  const int total_rows = a.num_blocks * a.num_kv_heads * B;
  uint32_t bad_mask = 0;  // bit st: the tile in stage st had an invalid block id

  // Warp-wide: fetch tile i into stage i % NSTAGE.
  auto issue = [&](int i) {
    if (i - win_base >= 32) {
      win_base += 32;
      const int k = win_base + lane;
      win_id = k < nt_w ? bt[tile_tok0(k) / B] : -1;
    }
    const int phys = __shfl_sync(FULL_MASK, win_id, i - win_base);
    const int st = i % NSTAGE;
    const bool bad = phys < 0 || phys >= a.num_blocks;
    bad_mask = bad ? (bad_mask | (1u << st)) : (bad_mask & ~(1u << st));
    if (lane == 0) {
      int y;
      if (bad) {
        report(a.err, PKV_DEV_BAD_BLOCK);
        y = total_rows;  // wholly out of bounds: TMA fills zeros
      } else {
        y = (phys * a.num_kv_heads + h) * B + (tile_tok0(i) % B);
      }
      const uint32_t bar = bar0 + 8 * st;
      const uint32_t kdst = ring + st * Shape::STAGE_BYTES;
      const uint32_t vdst = kdst + Shape::KT_BYTES;
      fence_proxy_async_smem();
      mbar_arrive_expect_tx(bar, Shape::STAGE_BYTES);
#pragma unroll
      for (int hh = 0; hh < Shape::HALVES; ++hh) {
        tma_load_2d(kdst + hh * HALF_BYTES, &tmK, hh * BOX_COLS, y, bar);
        tma_load_2d(vdst + hh * HALF_BYTES, &tmV, hh * BOX_COLS, y, bar);
      }
    }
  };

  float acc[D / 16][4];
#pragma unroll
  for (int mt = 0; mt < D / 16; ++mt) acc[mt][0] = acc[mt][1] = acc[mt][2] = acc[mt][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY;  // running max of heads 2c, 2c+1 (base-2 units)
  float l0 = 0.f, l1 = 0.f;              // this lane's share of the running sums
  const float sl2 = a.scale_log2;

  const int pre = nt_w < NSTAGE ? nt_w : NSTAGE;
  for (int i = 0; i < pre; ++i) issue(i);

  // ldmatrix.trans row addresses for V: lane feeds row (lane & 7) of matrix lane >> 3.
  const int mi = lane >> 3;
  const int vr = (lane & 7) + ((mi >> 1) << 3);  // token row inside the tile

  // A wait that gives up (never expected: a TMA load completes in microseconds)
  // ends this warp's loop with an error status instead of spinning on. CTAs
  // that start after such a report skip their waits too, so a failure cannot
  // turn into a long stall.
  bool aborted = a.err != nullptr &&
                 *reinterpret_cast<volatile const int32_t *>(a.err) == PKV_DEV_WAIT_TIMEOUT;

  for (int i = 0; i < nt_w && !aborted; ++i) {
    const int st = i % NSTAGE;
    const uint32_t bar = bar0 + 8 * st;
    const uint32_t parity = (i / NSTAGE) & 1;
    const bool ok = __all_sync(FULL_MASK, mbar_wait_bounded(bar, parity));
    if (!ok) {
      if (lane == 0) report(a.err, PKV_DEV_WAIT_TIMEOUT);
      aborted = true;
      break;
    }
    const uint32_t ks = ring + st * Shape::STAGE_BYTES;
    const uint32_t vs = ks + Shape::KT_BYTES;
    const int tok0 = tile_tok0(i);
    const int valid = min(TILE, L - tok0);
    const bool bad = (bad_mask >> st) & 1u;

    if (valid < TILE && !bad) {
      // Tokens past the context length: their V rows may hold anything
      // (NaN included); zero them so P*V stays finite.
      const int nchunks = (TILE - valid) * 8 * Shape::HALVES;
      for (int e = lane; e < nchunks; e += 32) {
        const int r = valid + e / (8 * Shape::HALVES);
        const int rem = e % (8 * Shape::HALVES);
        sts128_zero(vs + (rem >> 3) * HALF_BYTES + r * 128 + (rem & 7) * 16);
      }
      __syncwarp();
    }

    // ---- scores: S^T = K . Q^T ----
    float sc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int j = 0; j < D / 32; ++j) {
      const int Lc = (j >> 1) * 8 + 2 * c + (j & 1);
      const uint32_t rowg = ks + (Lc >> 3) * HALF_BYTES + g * 128 + (((Lc & 7) ^ g) << 4);
      const uint4 ka = lds128(rowg);             // token g
      const uint4 kb = lds128(rowg + 8 * 128);   // token g + 8 (same swizzle phase)
      mma16816<T>(sc, ka.x, kb.x, ka.y, kb.y, qf[j].x, qf[j].y);
      mma16816<T>(sc, ka.z, kb.z, ka.w, kb.w, qf[j].z, qf[j].w);
    }

    // ---- online softmax (heads 2c, 2c+1; tokens g, g+8) ----
    const bool ok0 = !bad && g < valid;
    const bool ok1 = !bad && g + 8 < valid;
    const float x0 = ok0 ? sc[0] * sl2 : -INFINITY;
    const float x1 = ok0 ? sc[1] * sl2 : -INFINITY;
    const float x2 = ok1 ? sc[2] * sl2 : -INFINITY;
    const float x3 = ok1 ? sc[3] * sl2 : -INFINITY;
    float mx0 = fmaxf(x0, x2), mx1 = fmaxf(x1, x3);
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      mx0 = fmaxf(mx0, __shfl_xor_sync(FULL_MASK, mx0, off));
      mx1 = fmaxf(mx1, __shfl_xor_sync(FULL_MASK, mx1, off));
    }
    const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
    const float mu0 = mn0 == -INFINITY ? 0.f : mn0;
    const float mu1 = mn1 == -INFINITY ? 0.f : mn1;
    const float al0 = ex2_approx(m0 - mu0), al1 = ex2_approx(m1 - mu1);
    const float p0 = ex2_approx(x0 - mu0), p1 = ex2_approx(x1 - mu1);
    const float p2 = ex2_approx(x2 - mu0), p3 = ex2_approx(x3 - mu1);
    l0 = l0 * al0 + (p0 + p2);
    l1 = l1 * al1 + (p1 + p3);
    m0 = mn0;
    m1 = mn1;
#pragma unroll
    for (int mt = 0; mt < D / 16; ++mt) {
      acc[mt][0] *= al0;
      acc[mt][1] *= al1;
      acc[mt][2] *= al0;
      acc[mt][3] *= al1;
    }

    // P^T as the B operand: transpose the (token, head) fragment pairs.
    const uint32_t pb0 = movmatrix_trans(pack2<T>(p0, p1));  // tokens 0..7
    const uint32_t pb1 = movmatrix_trans(pack2<T>(p2, p3));  // tokens 8..15

    // ---- O^T += V^T . P^T ----
    const uint32_t vrow = vs + vr * 128;
#pragma unroll
    for (int mt = 0; mt < D / 16; ++mt) {
      const int chunk = 2 * mt + (mi & 1);
      const uint32_t addr = vrow + (chunk >> 3) * HALF_BYTES + (((chunk & 7) ^ (vr & 7)) << 4);
      uint32_t r0, r1, r2, r3;
      ldsm_x4_trans(addr, r0, r1, r2, r3);
      mma16816<T>(acc[mt], r0, r1, r2, r3, pb0, pb1);
    }
    __syncwarp();
    if (i + NSTAGE < nt_w) issue(i + NSTAGE);
  }

  // Full per-warp sums: add the 8 lanes that share a head pair.
#pragma unroll
  for (int off = 4; off < 32; off <<= 1) {
    l0 += __shfl_xor_sync(FULL_MASK, l0, off);
    l1 += __shfl_xor_sync(FULL_MASK, l1, off);
  }

  // ---- combine the warps (their rings are idle now: every issued tile was consumed) ----
  __syncthreads();
  constexpr int AS = Shape::ACC_STRIDE;
  {
    float *cw = reinterpret_cast<float *>(smem_gen + warp * NSTAGE * Shape::STAGE_BYTES);
#pragma unroll
    for (int mt = 0; mt < D / 16; ++mt) {
      cw[(2 * c) * AS + 16 * mt + g] = acc[mt][0];
      cw[(2 * c + 1) * AS + 16 * mt + g] = acc[mt][1];
      cw[(2 * c) * AS + 16 * mt + g + 8] = acc[mt][2];
      cw[(2 * c + 1) * AS + 16 * mt + g + 8] = acc[mt][3];
    }
    if (g == 0) {
      cw[8 * AS + 2 * c] = m0;
      cw[8 * AS + 2 * c + 1] = m1;
      cw[8 * AS + 8 + 2 * c] = l0;
      cw[8 * AS + 8 + 2 * c + 1] = l1;
    }
  }
  __syncthreads();

  const bool single = nparts == 1;
  for (int idx = threadIdx.x; idx < G * D; idx += NWARPS * 32) {
    const int n = idx / D;
    const int d = idx - n * D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < NWARPS; ++w) {
      const float *cw = reinterpret_cast<const float *>(smem_gen + w * NSTAGE * Shape::STAGE_BYTES);
      M = fmaxf(M, cw[8 * AS + n]);
    }
    float num = 0.f, den = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < NWARPS; ++w) {
        const float *cw =
            reinterpret_cast<const float *>(smem_gen + w * NSTAGE * Shape::STAGE_BYTES);
        const float f = exp2f(cw[8 * AS + n] - M);
        num += f * cw[n * AS + d];
        den += f * cw[8 * AS + 8 + n];
      }
    }
    const float o = den > 0.f ? num / den : 0.f;
    const size_t row = (size_t)s * Hq + h * G + n;
    if (single) {
      out[row * D + d] = from_float<T>(o);
    } else {
      a.ws_o[(row * a.max_parts + p) * D + d] = o;
      if (d == 0) a.ws_lse[row * a.max_parts + p] = den > 0.f ? M + log2f(den) : -INFINITY;
    }
  }
}

template <typename T, int D>
cudaError_t launch_tc(const DecodeArgs &a, const CUtensorMap &tmK, const CUtensorMap &tmV,
                      cudaStream_t stream) {
  using Shape = TcShape<D>;
  auto kern = decode_tc_kernel<T, D>;
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Shape::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  dim3 grid(a.max_parts, a.num_kv_heads, a.num_seqs);
  kern<<<grid, NWARPS * 32, Shape::SMEM_BYTES, stream>>>(tmK, tmV, a);
  return cudaGetLastError();
}

}  // namespace

size_t decode_tc_smem_bytes(int head_dim) {
  return head_dim == 64 ? TcShape<64>::SMEM_BYTES : TcShape<128>::SMEM_BYTES;
}

cudaError_t launch_decode_tc(const DecodeArgs &a, int dtype, const CUtensorMap &tmK,
                             const CUtensorMap &tmV, cudaStream_t stream) {
  if (dtype == PKV_BF16) {
    if (a.head_dim == 64) return launch_tc<__nv_bfloat16, 64>(a, tmK, tmV, stream);
    return launch_tc<__nv_bfloat16, 128>(a, tmK, tmV, stream);
  }
  if (a.head_dim == 64) return launch_tc<__half, 64>(a, tmK, tmV, stream);
  return launch_tc<__half, 128>(a, tmK, tmV, stream);
}

}  // namespace pkv
