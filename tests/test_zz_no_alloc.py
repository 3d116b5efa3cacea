"""paged_attn_decode_static_ws: the decode entry point that allocates nothing.

It serves callers that must not allocate device memory while they decode, for
example an engine that gave nearly all GPU memory to its KV block pool at
start-up. Its workspace comes from a fixed 64 MiB array inside the library.
This test calls it through the C ABI twice in a row. Each time its output
must match the allocating entry point's, within the tolerance the parity
tests use. It also checks that a request too big for the array is refused
before anything is launched.

The file name makes pytest collect it last, so a run that stops at the first
failure has already run every other test.
"""

import ctypes

import numpy as np
import pytest
import torch

import paged_kv_cache_387_b200 as pkv
from pkv_inputs import make_random_case
from tests.helpers import TOL_16

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


def test_static_workspace_decode_matches_allocating_decode_twice():
    fn = _static_fn()
    # split contexts (up to 2000 tokens in 64-token partitions, two merge levels)
    c = make_random_case("noalloc", 32, 8, 128, 16, [1, 15, 300, 511, 512, 2000, 1337, 64],
                         torch.bfloat16, seed=77, device="cuda")
    need = pkv.decode_workspace_bytes(c.num_seqs, c.num_heads, c.head_dim,
                                      c.max_context_len, 64)
    assert 0 < need <= STATIC_WS_BYTES
    ref = torch.empty_like(c.q)
    pkv.paged_attn_decode(ref, c.q, c.k_pool, c.v_pool, c.block_tables, c.context_lens,
                          c.scale, c.max_context_len, partition_size=64)
    a, r = TOL_16
    for _ in range(2):
        out = torch.full_like(c.q, float("nan"))
        assert _call(fn, out, c, 64) == pkv.PKV_OK
        torch.cuda.synchronize()
        g = out.double().cpu().numpy()
        e = ref.double().cpu().numpy()
        assert not np.isnan(g).any()
        assert (np.abs(g - e) <= a + r * np.abs(e)).all()


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
