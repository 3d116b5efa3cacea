// Cache-append and block-copy kernels: byte-exact 16-byte vector moves.
//
// Append follows page "PagedAttention 논문 쉽게 읽기" (iplexlaw.co.kr),
// section 2: a new token's K/V go into the free slot of its sequence's last
// block. The slot is given by the slot mapping (phys_block * block_size +
// offset).
//
// Block copy is the data half of copy-on-write (page "추론 엔진에서의 메모리
// 가상화", molayo1419.me, copy-on-write section): a block shared by several
// sequences is copied whole before one of them writes into it.
//
// Block swap is the data half of swapping (page "PagedAttention Analysis",
// ryotta.opik.net, section 6): a preempted sequence's blocks are copied to
// CPU memory under a CPU block allocator, and copied back when it resumes.
#include "pkv_device.cuh"
#include "pkv_internal.h"

namespace pkv {
namespace {

constexpr int CACHE_THREADS = 256;

__global__ void __launch_bounds__(CACHE_THREADS)
    append_kernel(uint4 *__restrict__ kp, uint4 *__restrict__ vp, const uint4 *__restrict__ kn,
                  const uint4 *__restrict__ vn, const int64_t *__restrict__ slots, int T,
                  int Hkv, int vpr, int B, int num_blocks, int32_t *err) {
  const long long total = (long long)T * Hkv * vpr;
  const long long limit = (long long)num_blocks * B;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const long long row = i / vpr;  // token * Hkv + head
    const int v = (int)(i - row * vpr);
    const int t = (int)(row / Hkv);
    const int hh = (int)(row - (long long)t * Hkv);
    const long long slot = slots[t];
    if (slot < 0) continue;
    if (slot >= limit) {
      report(err, PKV_DEV_BAD_SLOT);
      continue;
    }
    const long long blk = slot / B;
    const int off = (int)(slot - blk * B);
    const long long dst = ((blk * Hkv + hh) * B + off) * vpr + v;
    kp[dst] = kn[i];
    vp[dst] = vn[i];
  }
}

constexpr int COPY_UNROLL = 4;

// Whole-block moves: for each pair (src, dst) the K and V slices of block src
// of the source pools are copied into block dst of the destination pools. The
// pools may be the same (copy-on-write inside the device pool) or different,
// e.g. the device pool and a swap space in page-locked host memory that the
// device addresses directly. Each thread keeps COPY_UNROLL 16-byte vectors of
// K and of V in flight, which is what a read over the host link needs.
__global__ void __launch_bounds__(CACHE_THREADS)
    block_move_kernel(uint4 *__restrict__ kd, uint4 *__restrict__ vd,
                      const uint4 *__restrict__ ks, const uint4 *__restrict__ vs,
                      const int32_t *__restrict__ pairs, int num_pairs, long long vpb,
                      int src_blocks, int dst_blocks, int32_t *err) {
  for (int pr = blockIdx.y; pr < num_pairs; pr += gridDim.y) {
    const int src = pairs[2 * pr];
    const int dst = pairs[2 * pr + 1];
    if (src < 0 || src >= src_blocks || dst < 0 || dst >= dst_blocks) {
      if (threadIdx.x == 0 && blockIdx.x == 0) report(err, PKV_DEV_BAD_PAIR);
      continue;
    }
    const uint4 *kb = ks + (long long)src * vpb;
    const uint4 *vb = vs + (long long)src * vpb;
    uint4 *kt = kd + (long long)dst * vpb;
    uint4 *vt = vd + (long long)dst * vpb;
    const long long stride = (long long)gridDim.x * blockDim.x * COPY_UNROLL;
    for (long long base = (long long)blockIdx.x * blockDim.x * COPY_UNROLL; base < vpb;
         base += stride) {
      uint4 rk[COPY_UNROLL], rv[COPY_UNROLL];
#pragma unroll
      for (int u = 0; u < COPY_UNROLL; ++u) {
        const long long i = base + (long long)u * blockDim.x + threadIdx.x;
        if (i < vpb) {
          rk[u] = kb[i];
          rv[u] = vb[i];
        }
      }
#pragma unroll
      for (int u = 0; u < COPY_UNROLL; ++u) {
        const long long i = base + (long long)u * blockDim.x + threadIdx.x;
        if (i < vpb) {
          kt[i] = rk[u];
          vt[i] = rv[u];
        }
      }
    }
  }
}

cudaError_t launch_block_move(void *kd, void *vd, const void *ks, const void *vs,
                              const int32_t *pairs, int num_pairs, long long block_bytes,
                              int src_blocks, int dst_blocks, int32_t *err, cudaStream_t stream) {
  const long long vpb = block_bytes / 16;
  long long gx = (vpb + (long long)CACHE_THREADS * COPY_UNROLL - 1) /
                 ((long long)CACHE_THREADS * COPY_UNROLL);
  if (gx > 64) gx = 64;
  const int gy = num_pairs < 65535 ? num_pairs : 65535;
  dim3 grid((unsigned)gx, (unsigned)gy);
  block_move_kernel<<<grid, CACHE_THREADS, 0, stream>>>(
      static_cast<uint4 *>(kd), static_cast<uint4 *>(vd), static_cast<const uint4 *>(ks),
      static_cast<const uint4 *>(vs), pairs, num_pairs, vpb, src_blocks, dst_blocks, err);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_append(void *k_pool, void *v_pool, const void *k_new, const void *v_new,
                          const int64_t *slots, int num_tokens, int num_kv_heads, int row_bytes,
                          int block_size, int num_blocks, int32_t *err, cudaStream_t stream) {
  const int vpr = row_bytes / 16;
  const long long total = (long long)num_tokens * num_kv_heads * vpr;
  long long blocks = (total + CACHE_THREADS - 1) / CACHE_THREADS;
  if (blocks > 148LL * 16) blocks = 148LL * 16;
  append_kernel<<<(unsigned)blocks, CACHE_THREADS, 0, stream>>>(
      static_cast<uint4 *>(k_pool), static_cast<uint4 *>(v_pool),
      static_cast<const uint4 *>(k_new), static_cast<const uint4 *>(v_new), slots, num_tokens,
      num_kv_heads, vpr, block_size, num_blocks, err);
  return cudaGetLastError();
}

cudaError_t launch_block_copy(void *k_pool, void *v_pool, const int32_t *pairs, int num_pairs,
                              long long block_bytes, int num_blocks, int32_t *err,
                              cudaStream_t stream) {
  return launch_block_move(k_pool, v_pool, k_pool, v_pool, pairs, num_pairs, block_bytes,
                           num_blocks, num_blocks, err, stream);
}

cudaError_t launch_block_swap(void *dst_k, void *dst_v, const void *src_k, const void *src_v,
                              const int32_t *pairs, int num_pairs, long long block_bytes,
                              int src_blocks, int dst_blocks, int32_t *err, cudaStream_t stream) {
  return launch_block_move(dst_k, dst_v, src_k, src_v, pairs, num_pairs, block_bytes, src_blocks,
                           dst_blocks, err, stream);
}

}  // namespace pkv
