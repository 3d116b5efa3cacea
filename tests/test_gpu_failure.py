"""Failure detection without a GPU fault. Every wait of the decode kernels is
bounded: a wait that gives up reports PKV_DEV_WAIT_TIMEOUT and the kernel
returns; a decode started after such a report does no work. The context stays
usable throughout."""

import time

import pytest
import torch

import oracle
import paged_kv_cache_387_b200 as pkv
from pkv_inputs import make_random_case
from tests.helpers import assert_close_to_oracle, gpu_decode, new_err, oracle_decode

pytestmark = pytest.mark.gpu
DEV = "cuda"
TIMEOUT = 5  # PKV_DEV_WAIT_TIMEOUT


@pytest.fixture(autouse=True, params=["auto", "persistent"])
def _dispatch(request):
    """Both decode kernels: the single-wave one (these calls are small) and
    the persistent one."""
    if request.param == "persistent":
        pkv.set_decode_dispatch(pkv.DISPATCH_PERSISTENT)
    yield
    pkv.set_decode_dispatch(pkv.DISPATCH_AUTO)


def test_bounded_wait_gives_up_and_reports():
    err = new_err(DEV)
    t0 = time.time()
    pkv.check_wait_timeout(err, limit_cycles=2_000_000)  # about a millisecond
    torch.cuda.synchronize()
    assert int(err.item()) == TIMEOUT
    assert time.time() - t0 < 10
    # the context is still usable
    c = make_random_case("after", 8, 2, 128, 16, [1, 40, 300], torch.bfloat16, seed=4,
                         device=DEV)
    assert_close_to_oracle(gpu_decode(c), oracle_decode(c), torch.bfloat16, "after timeout")


def test_decode_after_a_timeout_report_does_no_work():
    c = make_random_case("stale", 8, 2, 128, 16, [40, 300, 5, 2100], torch.bfloat16, seed=3,
                         device=DEV, with_append=True)
    kp0, vp0 = c.k_pool.clone(), c.v_pool.clone()
    err = torch.full((1,), TIMEOUT, dtype=torch.int32, device=DEV)
    out = torch.full_like(c.q, 7.0)
    pkv.paged_attn_decode_append(out, c.q, c.k_new, c.v_new, c.k_pool, c.v_pool, c.block_tables,
                                 c.context_lens, c.scale, c.max_context_len, partition_size=512,
                                 err=err)
    pkv.paged_attn_decode(out, c.q, c.k_pool, c.v_pool, c.block_tables, c.context_lens, c.scale,
                          c.max_context_len, partition_size=512, err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == TIMEOUT
    assert (out == 7.0).all()  # nothing written
    assert torch.equal(c.k_pool.view(torch.int16), kp0.view(torch.int16))  # nothing appended
    assert torch.equal(c.v_pool.view(torch.int16), vp0.view(torch.int16))
    # once the word is reset, the same call works
    err.zero_()
    pkv.paged_attn_decode_append(out, c.q, c.k_new, c.v_new, c.k_pool, c.v_pool, c.block_tables,
                                 c.context_lens, c.scale, c.max_context_len, partition_size=512,
                                 err=err)
    kc, vc = kp0.cpu(), vp0.cpu()
    oracle.cache_append(kc, vc, c.k_new.cpu(), c.v_new.cpu(), c.slot_mapping.cpu())
    ref = oracle.paged_decode(c.q.cpu(), kc, vc, c.block_tables.cpu(), c.context_lens.cpu(),
                              c.scale)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert_close_to_oracle(out, ref, torch.bfloat16, "after reset")
