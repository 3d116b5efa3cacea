"""Tail-split work items against the oracle.

The persistent decode hands out its work items in list order, so the last
`items mod grid` items run while the rest of the grid has nothing left to do.
When that remainder is at most half the grid and those items are long, the
plan splits each of them into several pieces of consecutive tiles, and the
pieces' partial results are combined by log-sum-exp, as the split-context
step of page "PagedAttention Analysis", section 3, combines partitions. The
split is taken with one or two query heads per KV head (the layout whose
items may carry a group of sequences that share a prefix), never with more. The
result must still be each sequence's own causal attention (page
"PagedAttention", newikis, section "Mathematical formulation"): every output
is compared with the oracle. The plan's decision is read back from the
workspace's scheduling words: word 2 is the first tail item, word 3 the
pieces per tail item.
"""

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_387_b200 as pkv
from pkv_inputs import make_random_case, make_sharing_case
from tests.helpers import assert_close_to_oracle, new_err

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(autouse=True)
def persistent_kernel():
    """These calls are sized for the persistent kernel; keep them there."""
    pkv.set_decode_dispatch(pkv.DISPATCH_PERSISTENT)
    yield
    pkv.set_decode_dispatch(pkv.DISPATCH_AUTO)


def grid_ctas():
    # two CTAs per SM (the kernel's shared-memory plan)
    return 2 * torch.cuda.get_device_properties(0).multi_processor_count


def run(c, part, fused):
    """The decode (fused append or append + decode) on the CUDA path, the
    oracle's result, and the scheduling words the plan left."""
    kc, vc = c.k_pool.cpu(), c.v_pool.cpu()
    if c.k_new is not None:
        oracle.cache_append(kc, vc, c.k_new.cpu(), c.v_new.cpu(), c.slot_mapping.cpu())
    ref = oracle.paged_decode(c.q.cpu(), kc, vc, c.block_tables.cpu(), c.context_lens.cpu(),
                              c.scale)
    nbytes = pkv.decode_workspace_bytes(c.num_seqs, c.num_heads, c.head_dim, c.max_context_len,
                                        part)
    ws = torch.zeros(nbytes, dtype=torch.uint8, device=DEV)
    out = torch.empty_like(c.q)
    err = new_err(DEV)
    if fused:
        pkv.paged_attn_decode_append(out, c.q, c.k_new, c.v_new, c.k_pool, c.v_pool,
                                     c.block_tables, c.context_lens, c.scale, c.max_context_len,
                                     partition_size=part, workspace=ws, err=err)
    else:
        if c.k_new is not None:
            pkv.kv_cache_append(c.k_pool, c.v_pool, c.k_new, c.v_new, c.slot_mapping, err=err)
        pkv.paged_attn_decode(out, c.q, c.k_pool, c.v_pool, c.block_tables, c.context_lens,
                              c.scale, c.max_context_len, partition_size=part, workspace=ws,
                              err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    if c.k_new is not None:
        assert torch.equal(c.k_pool.cpu().view(torch.int16), kc.view(torch.int16))
        assert torch.equal(c.v_pool.cpu().view(torch.int16), vc.view(torch.int16))
    words = ws[:16].view(torch.int32).cpu().tolist()
    return out, ref, words


def last_entry_tiles(lens, part):
    """Tiles of the work list's last entry: the one-partition sequences are
    ordered by 64 size classes, largest first, batch order within a class."""
    max_tiles = part // 16
    best = None
    for s, n in enumerate(lens):
        t = -(-n // 16)
        if t > max_tiles:
            continue  # several partitions: listed ahead of the classes
        b = 63 - min(63, t * 63 // max_tiles)
        if best is None or b >= best[0]:
            best = (b, t)
    return best[1]


def expected_split(items, smallest_tiles, G, slots=512):
    """The plan's rule, restated: (first tail item, pieces) or (0, 0)."""
    grid = grid_ctas()
    if G > 2:
        return 0, 0
    r = items % grid
    if items <= grid or r == 0:
        return 0, 0
    k = min(8, grid // r, slots // r, smallest_tiles // 8)
    return (items - r, k) if k >= 2 else (0, 0)


@pytest.mark.parametrize("dt", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("Hq,Hkv", [(8, 8), (16, 8)])
@pytest.mark.parametrize("D,B", [(128, 16), (64, 8)])
@pytest.mark.parametrize("fused", [False, True])
def test_one_sequence_items(dt, Hq, Hkv, D, B, fused):
    """Sequences that share nothing (one sequence per item): 24 items past a
    whole wave, each split into up to 8 pieces."""
    S = (grid_ctas() + 24) // Hkv
    rng = np.random.default_rng(7 + D + B)
    lens = rng.integers(700, 1400, size=S).tolist()
    c = make_random_case("tail1", Hq, Hkv, D, B, lens, dt, seed=11 + D, device=DEV,
                         with_append=True)
    out, ref, words = run(c, 2048, fused)
    want = expected_split(S * Hkv, last_entry_tiles(lens, 2048), Hq // Hkv)
    assert want[1] >= 2
    assert (words[2], words[3]) == want
    assert_close_to_oracle(out, ref, dt, f"tail split {dt} G{Hq // Hkv} D{D} B{B} f{fused}")


@pytest.mark.parametrize("Hq,Hkv", [(32, 8), (24, 8), (64, 8)])  # G = 4, 3, 8
def test_three_or_more_heads_per_kv_head_are_not_split(Hq, Hkv):
    S = (grid_ctas() + 24) // Hkv
    c = make_random_case("tailg4", Hq, Hkv, 128, 16, [1000] * S, torch.bfloat16, seed=13,
                         device=DEV, with_append=True)
    out, ref, words = run(c, 2048, True)
    assert words[3] == 0
    assert_close_to_oracle(out, ref, torch.bfloat16, f"G{Hq // Hkv}: no tail split")


@pytest.mark.parametrize("Hq,Hkv", [(8, 8), (16, 8)])  # G = 1 (8 members), G = 2 (4 members)
@pytest.mark.parametrize("D,B,dt", [(128, 16, torch.float16), (64, 24, torch.bfloat16)])
@pytest.mark.parametrize("fused", [False, True])
def test_shared_prefix_group_items(Hq, Hkv, D, B, dt, fused):
    """Groups of samples that share a prompt: the tail's group items are split,
    each piece covering part of the shared tiles or of the members' own ones.
    Block 24 puts the two 8-token halves of some tiles in different blocks."""
    members = 8 // (Hq // Hkv)
    n_groups = (grid_ctas() + 24) // Hkv
    rng = np.random.default_rng(5 + Hq + B)
    groups = [(int(rng.integers(400, 700)), [int(x) for x in rng.integers(1, 80, size=members)])
              for _ in range(n_groups)]
    c = make_sharing_case("tailg", Hq, Hkv, D, B, groups, dt, seed=21 + Hq + B, device=DEV,
                          with_append=True)
    out, ref, words = run(c, 2048, fused)
    assert words[3] >= 2, words  # the tail was split
    assert words[2] == n_groups * Hkv - n_groups * Hkv % grid_ctas()
    assert_close_to_oracle(out, ref, dt, f"tail split groups G{Hq // Hkv} D{D} B{B}")


def test_remainder_too_large_is_not_split():
    """A remainder above half the grid is left whole (the tail already keeps
    most of the grid busy)."""
    Hq, Hkv = 8, 8
    grid = grid_ctas()
    S = (grid + grid // 2 + 16) // Hkv
    c = make_random_case("tailno", Hq, Hkv, 128, 16, [900] * S, torch.bfloat16, seed=3,
                         device=DEV, with_append=True)
    out, ref, words = run(c, 2048, True)
    assert S * Hkv % grid > grid // 2
    assert words[3] == 0
    assert_close_to_oracle(out, ref, torch.bfloat16, "no tail split")


def test_short_items_are_not_split():
    """Items of fewer than 16 tiles cannot give two pieces of 8 tiles."""
    Hq, Hkv = 8, 8
    S = (grid_ctas() + 24) // Hkv
    c = make_random_case("tailshort", Hq, Hkv, 128, 16, [200] * S, torch.bfloat16, seed=4,
                         device=DEV, with_append=True)
    out, ref, words = run(c, 2048, True)
    assert words[3] == 0
    assert_close_to_oracle(out, ref, torch.bfloat16, "short items")


def test_split_items_beside_split_contexts():
    """Multi-partition sequences (1024-token partitions) ahead of the
    one-partition tail: both merges in one call."""
    Hq, Hkv = 8, 8
    S = (grid_ctas() + 24) // Hkv
    lens = [3000] * 4 + [900] * (S - 4)
    c = make_random_case("tailmix", Hq, Hkv, 128, 16, lens, torch.bfloat16, seed=9, device=DEV,
                         with_append=True)
    out, ref, words = run(c, 1024, True)
    items = (4 * 3 + (S - 4)) * Hkv
    assert (words[2], words[3]) == expected_split(items, last_entry_tiles(lens, 1024), 1)
    assert_close_to_oracle(out, ref, torch.bfloat16, "tail split beside split contexts")


def test_repeated_calls_reset_the_piece_counters():
    """The plan zeroes the piece counters on every call: the same workspace
    serves several calls in a row."""
    Hq, Hkv = 16, 8
    S = (grid_ctas() + 24) // Hkv
    c = make_random_case("tailrep", Hq, Hkv, 128, 16, [1100] * S, torch.bfloat16, seed=12,
                         device=DEV)
    ref = oracle.paged_decode(c.q.cpu(), c.k_pool.cpu(), c.v_pool.cpu(), c.block_tables.cpu(),
                              c.context_lens.cpu(), c.scale)
    nbytes = pkv.decode_workspace_bytes(S, Hq, 128, c.max_context_len, 2048)
    ws = torch.zeros(nbytes, dtype=torch.uint8, device=DEV)
    outs = [torch.empty_like(c.q) for _ in range(4)]
    err = new_err(DEV)
    for o in outs:
        pkv.paged_attn_decode(o, c.q, c.k_pool, c.v_pool, c.block_tables, c.context_lens,
                              c.scale, c.max_context_len, partition_size=2048, workspace=ws,
                              err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert ws[:16].view(torch.int32).cpu().tolist()[3] >= 2
    for o in outs:
        assert_close_to_oracle(o, ref, torch.bfloat16, "repeated tail split")
        assert torch.equal(o, outs[0])
