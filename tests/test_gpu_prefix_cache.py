"""Automatic prefix caching (page "PagedAttention Analysis", section 4): blocks
keyed by a hash of the whole prefix are shared through a global table. The
cache's hits must be exactly the full blocks whose token prefix was seen
before; the fused append + decode over the shared blocks must match the
oracle; and the same requests laid out in private blocks must decode to the same
values."""

import pytest
import torch

import oracle
import paged_kv_cache_387_b200 as pkv
from pkv_inputs import make_prefix_cache_case
from tests.helpers import assert_close_to_oracle, new_err

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("dt,B,Hq,Hkv,D", [(torch.bfloat16, 16, 8, 2, 128),
                                          (torch.float16, 8, 4, 4, 64)])
def test_prefix_cache_sharing_decode(dt, B, Hq, Hkv, D):
    c = make_prefix_cache_case(device=DEV, seed=5, num_requests=8, system_len=100, groups=2,
                               group_len=40, suffix_range=(20, 50), num_heads=Hq,
                               num_kv_heads=Hkv, head_dim=D, block_size=B, dtype=dt)
    m = c.meta
    seen, hits = set(), 0
    for toks in m["tokens"]:
        for j in range(len(toks) // B):
            p = tuple(toks[:(j + 1) * B])
            hits += p in seen
            seen.add(p)
    assert m["hits"] == hits and hits > 0
    assert m["blocks_in_use"] < m["blocks_unshared"]

    kc, vc = c.k_pool.cpu(), c.v_pool.cpu()
    err = new_err(DEV)
    out = torch.empty_like(c.q)
    mcl = int(c.context_lens.max())
    pkv.paged_attn_decode_append(out, c.q, c.k_new, c.v_new, c.k_pool, c.v_pool, c.block_tables,
                                 c.context_lens, c.scale, mcl, partition_size=64, err=err)
    oracle.cache_append(kc, vc, c.k_new.cpu(), c.v_new.cpu(), c.slot_mapping.cpu())
    ref = oracle.paged_decode(c.q.cpu(), kc, vc, c.block_tables.cpu(), c.context_lens.cpu(),
                              c.scale)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert torch.equal(c.k_pool.cpu().view(torch.int16), kc.view(torch.int16))
    assert torch.equal(c.v_pool.cpu().view(torch.int16), vc.view(torch.int16))
    assert_close_to_oracle(out, ref, dt, "prefix cache")

    # the same requests in private blocks: block i of the unshared layout is a
    # copy of the i-th table entry (kv_block_swap between two device pools)
    bt = c.block_tables.cpu()
    lens = c.context_lens.cpu().tolist()
    entries = [int(bt[s, j]) for s, L in enumerate(lens) for j in range(-(-L // B))]
    P2 = len(entries)
    k2 = torch.full((P2,) + tuple(c.k_pool.shape[1:]), float("nan"), dtype=dt, device=DEV)
    v2 = torch.full_like(k2, float("nan"))
    pairs = torch.tensor([[e, i] for i, e in enumerate(entries)], dtype=torch.int32, device=DEV)
    pkv.kv_block_swap(k2, v2, c.k_pool, c.v_pool, pairs, err=err)
    bt2 = torch.full_like(bt, -1)
    pos = 0
    for s, L in enumerate(lens):
        n = -(-L // B)
        bt2[s, :n] = torch.arange(pos, pos + n, dtype=torch.int32)
        pos += n
    out2 = torch.empty_like(c.q)
    pkv.paged_attn_decode(out2, c.q, k2, v2, bt2.to(DEV), c.context_lens, c.scale, mcl,
                          partition_size=64, err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    # Requests that share cached blocks are attended together when a KV head
    # serves at most 4 query heads (one work item reads each shared tile once),
    # so the summation order differs from the private layout's: both must match
    # the oracle. With larger groups both layouts run the same arithmetic.
    assert_close_to_oracle(out2, ref, dt, "prefix cache, private blocks")
    if Hq // Hkv > 4:
        assert torch.equal(out2.view(torch.int16), out.view(torch.int16))
