"""Shared-prefix work items against the oracle.

Sequences next to each other in the batch whose block tables start with the
same physical blocks (the samples of one prompt, beams, cached prefixes: page
"PagedAttention Analysis", section 4) are attended by one work item when a
KV head serves one or two query heads. The item reads each shared tile once
for all of them, and each member's own tiles for that member only. The
result must still be each sequence's own causal attention (page
"PagedAttention", newikis, section "Mathematical formulation"): every output
is compared with the oracle, which knows nothing of groups. With the append
fused in, the pools must equal the oracle's append bit for bit.
"""

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_387_b200 as pkv
from pkv_inputs import make_sharing_case
from tests.helpers import assert_close_to_oracle, new_err

pytestmark = pytest.mark.gpu
DEV = "cuda"
DT = {"f16": torch.float16, "bf16": torch.bfloat16}

# (prompt_len, own token counts of the members); a prompt of 0 shares nothing
GROUPS = [(100, [5, 30, 1, 200]), (37, [3, 70]), (16, [1] * 9), (0, [20, 40]),
          (300, list(range(1, 21))), (64, [16, 16, 32]), (15, [3, 3]), (999, [1, 64, 9])]


def run_both(c, part, fused):
    """GPU decode (fused append or append + decode) and the oracle's result."""
    kc, vc = c.k_pool.cpu(), c.v_pool.cpu()
    oracle.cache_append(kc, vc, c.k_new.cpu(), c.v_new.cpu(), c.slot_mapping.cpu())
    ref = oracle.paged_decode(c.q.cpu(), kc, vc, c.block_tables.cpu(), c.context_lens.cpu(),
                              c.scale)
    out = torch.empty_like(c.q)
    err = new_err(DEV)
    if fused:
        pkv.paged_attn_decode_append(out, c.q, c.k_new, c.v_new, c.k_pool, c.v_pool,
                                     c.block_tables, c.context_lens, c.scale, c.max_context_len,
                                     partition_size=part, err=err)
    else:
        pkv.kv_cache_append(c.k_pool, c.v_pool, c.k_new, c.v_new, c.slot_mapping, err=err)
        pkv.paged_attn_decode(out, c.q, c.k_pool, c.v_pool, c.block_tables, c.context_lens,
                              c.scale, c.max_context_len, partition_size=part, err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert torch.equal(c.k_pool.cpu().view(torch.int16), kc.view(torch.int16))
    assert torch.equal(c.v_pool.cpu().view(torch.int16), vc.view(torch.int16))
    return out, ref


@pytest.mark.parametrize("dt", ["f16", "bf16"])
@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (8, 4), (8, 2)])  # G = 1, 2 (grouped), 4
@pytest.mark.parametrize("D,B", [(128, 16), (64, 8), (128, 24), (64, 32)])
@pytest.mark.parametrize("part", [0, 64, 512, pkv.PARTITION_AUTO])
@pytest.mark.parametrize("fused", [False, True])
def test_shared_prefix_groups_match_oracle(dt, Hq, Hkv, D, B, part, fused):
    c = make_sharing_case("groups", Hq, Hkv, D, B, GROUPS, DT[dt], seed=D + B + Hq + Hkv,
                          device=DEV, with_append=True)
    out, ref = run_both(c, part, fused)
    assert_close_to_oracle(out, ref, DT[dt], f"{dt} G{Hq // Hkv} D{D} B{B} p{part} f{fused}")


@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (8, 4)])
def test_groups_across_plan_rounds(Hq, Hkv):
    """The plan works through the batch 256 sequences at a time, and groups do
    not cross those rounds: 50 prompts of 6 samples put one prompt's samples
    on both sides of sequence 256."""
    groups = [(200 + 7 * i, [1 + (i * 13 + j * 5) % 40 for j in range(6)]) for i in range(50)]
    c = make_sharing_case("rounds", Hq, Hkv, 128, 16, groups, torch.bfloat16, seed=3,
                          device=DEV, with_append=True)
    assert c.num_seqs == 300
    out, ref = run_both(c, 2048, True)
    assert_close_to_oracle(out, ref, torch.bfloat16, "groups across rounds")


def test_sharing_that_is_not_a_prefix():
    """Two sequences whose tables agree on blocks 0-4, differ at block 5 and
    point to the same physical blocks again at 6 and 7: the group shares
    blocks 0-4 only, and blocks 6 and 7 are read once per sequence."""
    c = make_sharing_case("nonprefix", 4, 4, 128, 16, [(64, [100, 120]), (0, [50])],
                          torch.float16, seed=9, device=DEV, with_append=True)
    pkv.kv_cache_append(c.k_pool, c.v_pool, c.k_new, c.v_new, c.slot_mapping)
    bt = c.block_tables.clone()
    bt[1, 4] = bt[0, 4]      # the common prefix grows to blocks 0-4
    bt[1, 5] = bt[2, 1]      # block 5 differs (a block of the third sequence)
    bt[1, 6:8] = bt[0, 6:8]  # blocks 6 and 7 in common again
    c.block_tables = bt.contiguous()
    ref = oracle.paged_decode(c.q.cpu(), c.k_pool.cpu(), c.v_pool.cpu(), bt.cpu(),
                              c.context_lens.cpu(), c.scale)
    for part in (0, 64):
        out = torch.empty_like(c.q)
        pkv.paged_attn_decode(out, c.q, c.k_pool, c.v_pool, c.block_tables, c.context_lens,
                              c.scale, c.max_context_len, partition_size=part)
        assert_close_to_oracle(out, ref, torch.float16, f"non-prefix sharing p{part}")


def test_identical_sequences_share_everything():
    """Sequences with the same table and length (a fork before its first
    write) are one group; the shared span stops at the last whole tile and
    the remaining tokens are read per member."""
    c = make_sharing_case("same", 8, 4, 128, 16, [(0, [75])], torch.bfloat16, seed=4,
                          device=DEV)
    S = 5
    q = torch.randn(S, 8, 128, device=DEV).to(torch.bfloat16)
    bt = c.block_tables.expand(S, -1).contiguous()
    lens = c.context_lens.expand(S).contiguous()
    ref = oracle.paged_decode(q.cpu(), c.k_pool.cpu(), c.v_pool.cpu(), bt.cpu(), lens.cpu(),
                              c.scale)
    for part in (0, 16, 64):
        out = torch.empty_like(q)
        pkv.paged_attn_decode(out, q, c.k_pool, c.v_pool, bt, lens, c.scale, 75,
                              partition_size=part)
        assert_close_to_oracle(out, ref, torch.bfloat16, f"identical p{part}")


def test_bad_block_id_in_a_shared_block():
    """An out-of-range id in the shared span (every member's table holds it)
    is reported once and masks that tile for every member."""
    c = make_sharing_case("badshared", 4, 4, 128, 16, [(160, [10, 20, 30])], torch.float16,
                          seed=5, device=DEV)
    bt = c.block_tables.clone()
    bt[:, 2] = c.num_blocks + 3
    err = new_err(DEV)
    out = torch.empty_like(c.q)
    pkv.paged_attn_decode(out, c.q, c.k_pool, c.v_pool, bt.contiguous(), c.context_lens,
                          c.scale, c.max_context_len, partition_size=0, err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 1
    assert not torch.isnan(out.float()).any()


def test_group_results_are_deterministic():
    c = make_sharing_case("det", 4, 4, 128, 16, GROUPS, torch.bfloat16, seed=8, device=DEV)
    outs = []
    for _ in range(3):
        o = torch.empty_like(c.q)
        pkv.paged_attn_decode(o, c.q, c.k_pool, c.v_pool, c.block_tables, c.context_lens,
                              c.scale, c.max_context_len, partition_size=64)
        outs.append(o)
    torch.cuda.synchronize()
    for o in outs[1:]:
        assert torch.equal(o.view(torch.int16), outs[0].view(torch.int16))
