"""paged_attn_decode_static_ws: the decode entry point that allocates nothing.

It serves callers that must not allocate device memory while they decode, for
example an engine that gave nearly all GPU memory to its KV block pool at
start-up. Its workspace comes from a fixed 64 MiB array inside the library.
These tests call it through the C ABI twice in a row. Both entry points run
the same kernels on the same inputs, so each call's output must equal the
allocating entry point's bit for bit (which is inside any tolerance the
parity tests use). Across the second call neither torch's allocator nor the
device's free memory may change. A request too big for the array is refused
before anything is launched, and a call with no sequences returns what the
allocating entry point returns for the same arguments.

The file name makes pytest collect it last, so a run that stops at the first
failure has already run every other test.
"""

import ctypes

import pytest
import torch

import paged_kv_cache_387_b200 as pkv
from pkv_inputs import make_random_case

pytestmark = pytest.mark.gpu

STATIC_WS_BYTES = 64 * 1024 * 1024


def _static_fn():
    lib = pkv.load_library()
    fn = lib.paged_attn_decode_static_ws
    P, I, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    fn.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, I, I, F, I, I, P, P]
    fn.restype = I
    return fn


def _call(fn, out, c, partition_size, max_context_len=None):
    mcl = c.max_context_len if max_context_len is None else max_context_len
    ptr = lambda t: ctypes.c_void_p(t.data_ptr())
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return fn(ptr(out), ptr(c.q), ptr(c.k_pool), ptr(c.v_pool), ptr(c.block_tables),
              ptr(c.context_lens), c.num_seqs, c.num_heads, c.num_kv_heads, c.head_dim,
              c.block_size, c.block_tables.shape[1], c.num_blocks, mcl, c.scale,
              pkv.DTYPE_CODES[c.q.dtype], partition_size, None, stream)


CASES = [
    # bf16 GQA, split contexts (up to 2000 tokens in 64-token partitions, two merge levels)
    ("bf16_split", 32, 8, 128, 16, [1, 15, 300, 511, 512, 2000, 1337, 64], torch.bfloat16, 64),
    # fp16 MHA, the library chooses the partition length
    ("f16_auto", 8, 8, 128, 16, [4096, 3, 900], torch.float16, pkv.PARTITION_AUTO),
    # fp32: the CUDA-core decode plus its separate merge kernel
    ("f32_split", 4, 2, 64, 16, [1, 15, 16, 37, 700], torch.float32, 128),
]


@pytest.mark.parametrize("name,Hq,Hkv,D,B,lens,dt,part", CASES, ids=[c[0] for c in CASES])
def test_static_workspace_decode_equals_allocating_decode_twice(name, Hq, Hkv, D, B, lens, dt,
                                                                part):
    fn = _static_fn()
    c = make_random_case("noalloc_" + name, Hq, Hkv, D, B, lens, dt, seed=77, device="cuda")
    need = pkv.decode_workspace_bytes(c.num_seqs, c.num_heads, c.head_dim,
                                      c.max_context_len, part)
    assert 0 < need <= STATIC_WS_BYTES
    ref = torch.empty_like(c.q)
    pkv.paged_attn_decode(ref, c.q, c.k_pool, c.v_pool, c.block_tables, c.context_lens,
                          c.scale, c.max_context_len, partition_size=part)
    outs = [torch.full_like(c.q, float("nan")) for _ in range(2)]
    torch.cuda.synchronize()
    for i, out in enumerate(outs):
        if i == 1:
            torch_bytes = torch.cuda.memory_allocated()
            free_bytes = torch.cuda.mem_get_info()[0]
        assert _call(fn, out, c, part) == pkv.PKV_OK
        torch.cuda.synchronize()
    # the second call allocated nothing, through torch or the driver
    assert torch.cuda.memory_allocated() == torch_bytes
    assert torch.cuda.mem_get_info()[0] == free_bytes
    bits = torch.int32 if dt == torch.float32 else torch.int16
    for out in outs:
        assert torch.equal(out.view(bits), ref.view(bits))


def test_static_workspace_with_no_sequences_matches_the_allocating_entry_point():
    fn = _static_fn()
    lib = pkv.load_library()
    c = make_random_case("noalloc_empty", 8, 2, 128, 16, [5], torch.bfloat16, seed=1,
                         device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    ptr = lambda t: ctypes.c_void_p(t.data_ptr())
    out = torch.empty_like(c.q)
    # (num_heads, num_kv_heads, partition_size): valid, a bad group, a bad partition
    for Hq, Hkv, part in ((8, 2, 64), (8, 3, 64), (8, 2, 24)):
        args = (ptr(out), ptr(c.q), ptr(c.k_pool), ptr(c.v_pool), ptr(c.block_tables),
                ptr(c.context_lens), 0, Hq, Hkv, 128, 16, c.block_tables.shape[1],
                c.num_blocks, c.max_context_len, c.scale, pkv.DTYPE_CODES[c.q.dtype], part)
        want = lib.paged_attn_decode(*args, None, 0, None, stream)
        assert fn(*args, None, stream) == want
    assert want == pkv.PKV_EINVAL


def test_static_workspace_refuses_requests_beyond_its_size():
    fn = _static_fn()
    c = make_random_case("noalloc_big", 8, 8, 128, 16, [16] * 64, torch.float16, seed=3,
                         device="cuda")
    # a host-side bound of 2^20 tokens per context would need far more than 64 MiB
    assert pkv.decode_workspace_bytes(c.num_seqs, c.num_heads, c.head_dim, 1 << 20,
                                      512) > STATIC_WS_BYTES
    out = torch.zeros_like(c.q)
    assert _call(fn, out, c, 512, max_context_len=1 << 20) == pkv.PKV_EUNSUPPORTED
    torch.cuda.synchronize()
    assert (out == 0).all()  # nothing was launched
