// Paged decode attention for fp32 inputs, and the split-context merge.
//
// fp32 inputs keep fp32 arithmetic end to end: no tensor-core rounding of K,
// V or P. One CTA (4 warps) attends one (sequence, KV head, partition) for up
// to SIMT_GMAX of the query heads that share the KV head (a group of more is
// split over several CTAs). Each warp walks every 4th token: it looks up the
// token's physical block in the block table, loads the token's K and V rows
// once (one vector per lane) for all its heads, forms each head's score with
// a warp-wide dot product and updates that head's running max / sum /
// output. That is the online walk of page "PagedAttention Analysis"
// (ryotta.opik.net), section 3, one token at a time. The warps are then
// combined in shared memory, head by head.
//
// The merge kernel combines the partitions of a split context. Partition p
// contributes its normalised output o_p with weight 2^(lse_p - lse), where
// lse_p is its base-2 log-sum-exp and lse = log2 sum_p 2^lse_p.
#include "pkv_device.cuh"
#include "pkv_internal.h"

namespace pkv {
namespace {

constexpr int SIMT_WARPS = 4;
constexpr int SIMT_GMAX = 8;  // query heads one CTA attends together

// E consecutive floats (E = 2 or 4) as one aligned vector load.
template <int E>
__device__ __forceinline__ void load_vec(const float *p, float (&v)[E]) {
  if constexpr (E == 4) {
    const float4 t = *reinterpret_cast<const float4 *>(p);
    v[0] = t.x;
    v[1] = t.y;
    v[2] = t.z;
    v[3] = t.w;
  } else {
    static_assert(E == 2, "head_dim 64 or 128");
    const float2 t = *reinterpret_cast<const float2 *>(p);
    v[0] = t.x;
    v[1] = t.y;
  }
}

template <int D>
__global__ void __launch_bounds__(SIMT_WARPS * 32) decode_simt_f32_kernel(const DecodeArgs a) {
  constexpr int E = D / 32;  // elements per lane
  __shared__ float red_acc[SIMT_WARPS][SIMT_GMAX][D];
  __shared__ float red_ml[SIMT_WARPS][SIMT_GMAX][2];

  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int p = blockIdx.x;
  const int s = blockIdx.z;
  const int Hq = a.num_heads;
  const int Hkv = a.num_kv_heads;
  const int G = Hq / Hkv;
  const int nchunk = (G + SIMT_GMAX - 1) / SIMT_GMAX;  // CTAs per KV head
  const int kvh = blockIdx.y / nchunk;
  const int h0 = kvh * G + (blockIdx.y - kvh * nchunk) * SIMT_GMAX;  // first query head
  const int ng = min(SIMT_GMAX, kvh * G + G - h0);                   // heads of this CTA
  const int B = a.block_size;

  const int L = effective_len(a.context_lens[s], a.max_context_len, a.max_blocks, B,
                              threadIdx.x == 0 ? a.err : nullptr);
  float *out = static_cast<float *>(a.out);
  const size_t row0 = (size_t)s * Hq + h0;  // row of head h0; head h0 + g is row0 + g
  if (L <= 0) {
    if (p == 0)
      for (int i = threadIdx.x; i < ng * D; i += SIMT_WARPS * 32) out[row0 * D + i] = 0.f;
    return;
  }
  const int t_begin = p * a.part_tokens;
  if (t_begin >= L) return;
  const int t_end = min(L, t_begin + a.part_tokens);
  const int nparts = (L + a.part_tokens - 1) / a.part_tokens;

  const float *q = static_cast<const float *>(a.q);
  float qv[SIMT_GMAX][E];
#pragma unroll
  for (int g = 0; g < SIMT_GMAX; ++g) {
    if (g < ng) {
      load_vec<E>(q + (row0 + g) * D + lane * E, qv[g]);
    } else {
#pragma unroll
      for (int e = 0; e < E; ++e) qv[g][e] = 0.f;
    }
  }

  const float *kp = static_cast<const float *>(a.k_pool);
  const float *vp = static_cast<const float *>(a.v_pool);
  const int32_t *bt = a.block_tables + (size_t)s * a.max_blocks;

  float m[SIMT_GMAX], l[SIMT_GMAX], acc[SIMT_GMAX][E];
#pragma unroll
  for (int g = 0; g < SIMT_GMAX; ++g) {
    m[g] = -INFINITY;
    l[g] = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) acc[g][e] = 0.f;
  }

  for (int t = t_begin + warp; t < t_end; t += SIMT_WARPS) {
    const int phys = bt[t / B];
    if (phys < 0 || phys >= a.num_blocks) {
      if (lane == 0) report(a.err, PKV_DEV_BAD_BLOCK);
      continue;
    }
    const size_t base = (((size_t)phys * Hkv + kvh) * B + (t % B)) * D + lane * E;
    float kv[E], vv[E];
    load_vec<E>(kp + base, kv);
    load_vec<E>(vp + base, vv);
    float dot[SIMT_GMAX];
#pragma unroll
    for (int g = 0; g < SIMT_GMAX; ++g) {
      dot[g] = 0.f;
#pragma unroll
      for (int e = 0; e < E; ++e) dot[g] = fmaf(qv[g][e], kv[e], dot[g]);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1)
#pragma unroll
      for (int g = 0; g < SIMT_GMAX; ++g)
        if (g < ng) dot[g] += __shfl_xor_sync(FULL_MASK, dot[g], off);
#pragma unroll
    for (int g = 0; g < SIMT_GMAX; ++g) {
      if (g >= ng) continue;
      const float x = dot[g] * a.scale_log2;
      const float mn = fmaxf(m[g], x);
      const float al = exp2f(m[g] - mn);
      const float pr = exp2f(x - mn);
      l[g] = l[g] * al + pr;
#pragma unroll
      for (int e = 0; e < E; ++e) acc[g][e] = fmaf(pr, vv[e], acc[g][e] * al);
      m[g] = mn;
    }
  }

#pragma unroll
  for (int g = 0; g < SIMT_GMAX; ++g) {
    if (g >= ng) continue;
#pragma unroll
    for (int e = 0; e < E; ++e) red_acc[warp][g][lane * E + e] = acc[g][e];
    if (lane == 0) {
      red_ml[warp][g][0] = m[g];
      red_ml[warp][g][1] = l[g];
    }
  }
  __syncthreads();

  for (int i = threadIdx.x; i < ng * D; i += SIMT_WARPS * 32) {
    const int g = i / D;
    const int d = i - g * D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < SIMT_WARPS; ++w) M = fmaxf(M, red_ml[w][g][0]);
    float num = 0.f, den = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < SIMT_WARPS; ++w) {
        const float f = exp2f(red_ml[w][g][0] - M);
        num += f * red_acc[w][g][d];
        den += f * red_ml[w][g][1];
      }
    }
    const float o = den > 0.f ? num / den : 0.f;
    const size_t row = row0 + g;
    if (nparts == 1) {
      out[row * D + d] = o;
    } else {
      a.ws_o[(row * a.max_parts + p) * D + d] = o;
      if (d == 0) a.ws_lse[row * a.max_parts + p] = den > 0.f ? M + log2f(den) : -INFINITY;
    }
  }
}

constexpr int MERGE_THREADS = 256;

__device__ __forceinline__ float block_reduce(float v, bool is_max, float *scratch) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const float o = __shfl_xor_sync(FULL_MASK, v, off);
    v = is_max ? fmaxf(v, o) : v + o;
  }
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  __syncthreads();
  if (lane == 0) scratch[warp] = v;
  __syncthreads();
  v = scratch[0];
  for (int w = 1; w < MERGE_THREADS / 32; ++w) v = is_max ? fmaxf(v, scratch[w]) : v + scratch[w];
  return v;
}

template <typename T, int D>
__global__ void __launch_bounds__(MERGE_THREADS) merge_kernel(const DecodeArgs a) {
  constexpr int V = D / 4;               // float4 per row
  constexpr int R = MERGE_THREADS / V;   // partition rows read concurrently
  __shared__ float scratch[MERGE_THREADS / 32];
  __shared__ float4 red[MERGE_THREADS];
  // A programmatic dependent of the decode grid that wrote the partials (a
  // plain stream-ordered launch otherwise): wait for it to complete.
  pdl_wait();

  const int hq = blockIdx.x;
  const int s = blockIdx.y;
  const int L = effective_len(a.context_lens[s], a.max_context_len, a.max_blocks, a.block_size,
                              nullptr);
  const int nparts = (L + a.part_tokens - 1) / a.part_tokens;
  if (nparts <= 1) return;  // written directly by the decode kernel

  const size_t row = (size_t)s * a.num_heads + hq;
  const float *lse = a.ws_lse + row * a.max_parts;
  const int tid = threadIdx.x;

  float mx = -INFINITY;
  for (int q = tid; q < nparts; q += MERGE_THREADS) mx = fmaxf(mx, lse[q]);
  mx = block_reduce(mx, true, scratch);
  float sum = 0.f;
  if (mx != -INFINITY)
    for (int q = tid; q < nparts; q += MERGE_THREADS) sum += exp2f(lse[q] - mx);
  sum = block_reduce(sum, false, scratch);

  const int r = tid / V, cv = tid - (tid / V) * V;
  const float4 *po = reinterpret_cast<const float4 *>(a.ws_o + row * a.max_parts * D);
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  if (mx != -INFINITY) {
#pragma unroll 4
    for (int q = r; q < nparts; q += R) {
      const float w = exp2f(lse[q] - mx);
      const float4 v = po[(size_t)q * V + cv];
      acc.x += w * v.x;
      acc.y += w * v.y;
      acc.z += w * v.z;
      acc.w += w * v.w;
    }
  }
  red[tid] = acc;
  __syncthreads();
  if (r == 0) {
    float4 t = red[cv];
    for (int rr = 1; rr < R; ++rr) {
      const float4 u = red[rr * V + cv];
      t.x += u.x;
      t.y += u.y;
      t.z += u.z;
      t.w += u.w;
    }
    const float inv = sum > 0.f ? 1.f / sum : 0.f;
    T *out = static_cast<T *>(a.out) + row * D + 4 * cv;
    out[0] = from_float<T>(t.x * inv);
    out[1] = from_float<T>(t.y * inv);
    out[2] = from_float<T>(t.z * inv);
    out[3] = from_float<T>(t.w * inv);
  }
}

template <typename T, int D>
cudaError_t launch_merge_t(const DecodeArgs &a, cudaStream_t stream) {
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.num_heads, a.num_seqs);
  cfg.blockDim = dim3(MERGE_THREADS);
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, merge_kernel<T, D>, a);
}

}  // namespace

cudaError_t launch_decode_simt_f32(const DecodeArgs &a, cudaStream_t stream) {
  const int G = a.num_heads / a.num_kv_heads;
  dim3 grid(a.max_parts, a.num_kv_heads * ((G + SIMT_GMAX - 1) / SIMT_GMAX), a.num_seqs);
  if (a.head_dim == 64)
    decode_simt_f32_kernel<64><<<grid, SIMT_WARPS * 32, 0, stream>>>(a);
  else
    decode_simt_f32_kernel<128><<<grid, SIMT_WARPS * 32, 0, stream>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_merge(const DecodeArgs &a, int dtype, cudaStream_t stream) {
  if (dtype == PKV_F32)
    return a.head_dim == 64 ? launch_merge_t<float, 64>(a, stream)
                            : launch_merge_t<float, 128>(a, stream);
  if (dtype == PKV_F16)
    return a.head_dim == 64 ? launch_merge_t<__half, 64>(a, stream)
                            : launch_merge_t<__half, 128>(a, stream);
  return a.head_dim == 64 ? launch_merge_t<__nv_bfloat16, 64>(a, stream)
                          : launch_merge_t<__nv_bfloat16, 128>(a, stream);
}

}  // namespace pkv
