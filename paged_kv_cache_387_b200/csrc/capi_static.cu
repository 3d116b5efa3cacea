// paged_attn_decode_static_ws: decode with library-owned scratch memory.
//
// Some callers cannot allocate device memory at the time they decode. A
// serving engine typically hands nearly all of the GPU's memory to its KV
// block pool at start-up, so a later cudaMalloc for a few megabytes of split
// workspace can fail, or would have to go around the engine's own allocator.
// Other hosts forbid allocation outside initialisation because cudaMalloc
// may synchronise the device and its latency is unpredictable. For them
// this entry point takes the decode workspace from a fixed array that lives
// in this file, instead of from the caller.
//
// The array has PKV_STATIC_WS_BYTES bytes. Each GPU on which this entry
// point is used holds its own copy, from the first call on that device until
// the process exits. Every call on a device shares that copy.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "pkv.h"

namespace {

// The scratch itself. In host code this name is only a stand-in for the
// symbol, not a device address: its device address comes from
// cudaGetSymbolAddress below, once per device.
static __device__ __align__(256) unsigned char pkv_static_scratch[PKV_STATIC_WS_BYTES];

constexpr int kMaxDevices = 128;
std::mutex g_mutex;
void *g_scratch_addr[kMaxDevices] = {};
unsigned long long g_scratch_ctx[kMaxDevices] = {};

// Unique id of the calling thread's current context, or 0 if it cannot be
// read. cudaDeviceReset destroys a device's primary context, and the array of
// the context created after it may sit at another address; a changed id
// tells the lookup below to ask again.
unsigned long long current_context_id() {
  using GetCurrent = CUresult (*)(CUcontext *);
  using GetId = CUresult (*)(CUcontext, unsigned long long *);
  static GetCurrent get_current = nullptr;
  static GetId get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<GetCurrent>(p);
    p = nullptr;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<GetId>(p);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr ||
      get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

// Device address of this device's scratch copy. It is looked up with
// cudaGetSymbolAddress on the first call made while the device is current,
// and again only if the device's context has changed since (after a
// cudaDeviceReset).
int scratch_for_current_device(void **addr) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return PKV_ECUDA;
  if (dev < 0 || dev >= kMaxDevices) return PKV_EUNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mutex);
  const unsigned long long ctx = current_context_id();  // 0 before the context exists
  if (g_scratch_addr[dev] == nullptr || ctx == 0 || ctx != g_scratch_ctx[dev]) {
    void *p = nullptr;
    // (this call also makes the device's primary context current)
    if (cudaGetSymbolAddress(&p, pkv_static_scratch) != cudaSuccess || p == nullptr)
      return PKV_ECUDA;
    g_scratch_addr[dev] = p;
    g_scratch_ctx[dev] = current_context_id();
  }
  *addr = g_scratch_addr[dev];
  return PKV_OK;
}

}  // namespace

extern "C" int paged_attn_decode_static_ws(void *out, const void *q, const void *k_pool,
                                           const void *v_pool, const int32_t *block_tables,
                                           const int32_t *context_lens, int num_seqs,
                                           int num_heads, int num_kv_heads, int head_dim,
                                           int block_size, int max_blocks_per_seq,
                                           int num_blocks, int max_context_len, float scale,
                                           int dtype, int partition_size, int32_t *err,
                                           void *stream) {
  // Nothing to decode (or a negative count): the ordinary entry point checks
  // the other arguments and returns the same status, without a workspace.
  if (num_seqs <= 0)
    return paged_attn_decode(out, q, k_pool, v_pool, block_tables, context_lens, num_seqs,
                             num_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq,
                             num_blocks, max_context_len, scale, dtype, partition_size, nullptr,
                             0, err, stream);
  const size_t need = pkv_decode_workspace_bytes(num_seqs, num_heads, head_dim, max_context_len,
                                                 partition_size);
  if (need > (size_t)PKV_STATIC_WS_BYTES) return PKV_EUNSUPPORTED;  // too big for the array
  void *ws = nullptr;
  const int rc = scratch_for_current_device(&ws);
  if (rc != PKV_OK) return rc;
  return paged_attn_decode(out, q, k_pool, v_pool, block_tables, context_lens, num_seqs,
                           num_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq,
                           num_blocks, max_context_len, scale, dtype, partition_size, ws,
                           (size_t)PKV_STATIC_WS_BYTES, err, stream);
}
