"""Host block allocator: the pages' copy-on-write example, the waste bound
and the byte-count helper, each against a cited golden fixture."""

import json
import os

import numpy as np
import pytest

from pkv_inputs import BlockAllocator, kv_bytes_per_token, make_shared_prefix_case

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def load(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


def test_cow_worked_example():
    g = load("cow_worked_example.json")
    B, P = g["block_size"], g["num_blocks"]
    others = [b for b in range(P) if b not in g["prompt_blocks"] + [g["next_free_block"]]]
    order = g["prompt_blocks"] + [g["next_free_block"]] + others
    alloc = BlockAllocator(P, B, free_order=order)
    a = alloc.new_sequence(g["prompt_tokens"])
    assert a.table == g["prompt_blocks"]
    b = alloc.fork(a)
    assert [alloc.refcount(x) for x in a.table] == [2, 2]
    exp = g["expected"]
    slot, cow = alloc.append_slot(a)
    assert (cow.src, cow.dst) == tuple(exp["copy"])
    assert a.table == exp["branch_a_table"]
    assert b.table == exp["branch_b_table"]
    assert slot == exp["branch_a_slot"]
    for blk, ref in exp["refcounts"].items():
        assert alloc.refcount(int(blk)) == ref
    # branch B is now the only owner of block 11 and writes in place
    slot_b, cow_b = alloc.append_slot(b)
    assert cow_b is exp["branch_b_copy_on_its_write"]
    assert slot_b == 11 * B + g["prompt_tokens"] % B


def test_waste_bounded_by_last_block():
    g = load("block_waste.json")
    B = g["block_size"]
    rng = np.random.default_rng(0)
    alloc = BlockAllocator(100000, B, free_order=rng.permutation(100000).tolist())
    wastes = []
    for L in rng.integers(1, 5000, size=2000):
        s = alloc.new_sequence(int(L))
        w = BlockAllocator.waste_slots(s, B)
        assert 0 <= w <= g["max_waste_tokens"]
        wastes.append(w)
        alloc.release(s)
    assert abs(np.mean(wastes) - g["mean_waste_tokens_uniform_lengths"]) < 0.5


def test_growth_allocates_only_when_last_block_full():
    alloc = BlockAllocator(8, 4)
    s = alloc.new_sequence(3)
    assert len(s.table) == 1
    slot, cow = alloc.append_slot(s)      # fills the 4th slot
    assert cow is None and len(s.table) == 1 and slot == s.table[0] * 4 + 3
    slot, cow = alloc.append_slot(s)      # block full -> new block
    assert cow is None and len(s.table) == 2 and slot == s.table[1] * 4


def test_release_returns_blocks_when_unreferenced():
    alloc = BlockAllocator(6, 16)
    a = alloc.new_sequence(20)
    b = alloc.fork(a)
    free0 = alloc.num_free
    alloc.release(a)
    assert alloc.num_free == free0           # still referenced by b
    alloc.release(b)
    assert alloc.num_free == 6
    with pytest.raises(ValueError):
        alloc.free(0)


def test_opt13b_bytes_per_token():
    g = load("opt13b_kv_bytes.json")
    n = kv_bytes_per_token(g["num_layers"], g["num_kv_heads"], g["head_dim"], g["elem_bytes"])
    assert n == g["expected_bytes_per_token"]
    assert n / 1024 == g["expected_kib_per_token"]
    lo, hi = g["expected_max_sequence_gb_range"]
    assert lo <= n * g["max_positions"] / 1e9 <= hi


def test_shared_prefix_copies_follow_refcount_rule():
    c = make_shared_prefix_case(num_prompts=2, samples=3, prompt_len=40, decode_steps=5,
                                num_heads=2, num_kv_heads=2, head_dim=64)
    # per prompt: samples-1 copies (the last writer owns the block alone)
    assert c.cow_pairs.shape == (2 * 2, 2)
    assert len(set(c.cow_pairs[:, 1].tolist())) == 4
    st = c.steps[-1]
    assert st["context_lens"].tolist() == [45] * 6
    # full prompt blocks stay shared across the samples of one prompt
    bt = st["block_tables"]
    assert (bt[0, :2] == bt[1, :2]).all() and (bt[0, :2] == bt[2, :2]).all()
    assert bt[0, 2] != bt[1, 2] != bt[2, 2]


# ---------------------------------------------------------------------------
# swapping (page "PagedAttention Analysis", section 6): a CPU block allocator
# beside the GPU one, all-or-nothing moves, swap space bounded by the GPU pool
# ---------------------------------------------------------------------------

from pkv_inputs import SwapSpace  # noqa: E402


def _sharing_pattern(seqs):
    """Which table positions hold the same block (the ids themselves may differ)."""
    ids = [b for sq in seqs for b in sq.table]
    first = {}
    return [first.setdefault(b, i) for i, b in enumerate(ids)]


def test_swap_space_is_bounded_by_the_gpu_pool():
    gpu = BlockAllocator(10, 16)
    with pytest.raises(ValueError):
        SwapSpace(gpu, 11)
    assert SwapSpace(gpu).cpu.num_blocks == 10


def test_swap_out_is_all_or_nothing():
    gpu = BlockAllocator(20, 16)
    sw = SwapSpace(gpu, 4)
    a = gpu.new_sequence(70)  # 5 blocks > 4 free in the swap space
    before = (list(a.table), gpu.num_free, sw.cpu.num_free)
    with pytest.raises(MemoryError):
        sw.swap_out([a])
    assert (a.table, gpu.num_free, sw.cpu.num_free) == before and not a.on_host


def test_swap_round_trip_keeps_sharing_and_refcounts():
    B = 16
    gpu = BlockAllocator(40, B, free_order=np.random.default_rng(5).permutation(40))
    sw = SwapSpace(gpu)
    prompt = gpu.new_sequence(40)  # 2 full blocks + 1 partial
    samples = [prompt] + [gpu.fork(prompt) for _ in range(2)]
    for sq in samples:  # each sample writes one token: copy-on-write of the partial block
        gpu.append_slot(sq)
    pattern = _sharing_pattern(samples)
    distinct = len(set(b for sq in samples for b in sq.table))
    gpu_free0 = gpu.num_free
    moves = sw.swap_out(samples)
    assert len(moves) == distinct and len({m.src for m in moves}) == distinct
    assert all(sq.on_host for sq in samples)
    assert gpu.num_free == gpu_free0 + distinct  # nothing else referenced them
    assert _sharing_pattern(samples) == pattern
    shared = samples[0].table[0]
    assert sw.cpu.refcount(shared) == 3  # one reference per table entry
    # the moves map each GPU block to the CPU block that replaced it
    m = {mv.src: mv.dst for mv in moves}
    assert len(set(m.values())) == distinct
    back = sw.swap_in(samples)
    assert len(back) == distinct and not any(sq.on_host for sq in samples)
    assert sw.cpu.num_free == sw.cpu.num_blocks and gpu.num_free == gpu_free0
    assert _sharing_pattern(samples) == pattern
    assert gpu.refcount(samples[1].table[0]) == 3


def test_swap_out_copies_blocks_still_referenced_outside_the_group():
    gpu = BlockAllocator(12, 16)
    sw = SwapSpace(gpu)
    a = gpu.new_sequence(32)
    b = gpu.fork(a)  # b stays on the GPU
    moves = sw.swap_out([a])
    assert len(moves) == 2
    assert [gpu.refcount(x) for x in b.table] == [1, 1]  # still owned by b
    assert gpu.num_free == 10
    with pytest.raises(ValueError):
        sw.swap_out([a])  # already on the host


def test_adopt_takes_over_existing_tables():
    gpu = BlockAllocator(8, 16)
    sq = gpu.adopt([5, 2], 20)
    assert gpu.num_free == 6 and gpu.refcount(5) == 1
    other = gpu.adopt([5], 3)  # a shared first block
    assert gpu.refcount(5) == 2 and other.table == [5]
    with pytest.raises(ValueError):
        gpu.adopt([1], 40)  # 40 tokens need 3 blocks


# ---------------------------------------------------------------------------
# beam search (page "PagedAttention Analysis", section 4): beams share the
# prompt and intermediate blocks; the sharing pattern changes every step
# ---------------------------------------------------------------------------

from pkv_inputs import BeamSearch  # noqa: E402


def test_beam_search_sharing_and_no_leaks():
    B, W = 16, 4
    alloc = BlockAllocator(200, B)
    bs = BeamSearch(alloc, prompt_tokens=40, width=W)
    rng = np.random.default_rng(3)
    for t in range(60):
        parents = rng.integers(0, W, size=W) if t % 7 else np.zeros(W, dtype=int)
        slots, copies = bs.step(parents)
        assert len(slots) == W and len(set(slots)) == W  # every beam writes its own slot
        for b in bs.beams:
            assert alloc.refcount(b.table[-1]) == 1  # the block being written is private
        # every block of a beam is referenced at least once per beam that holds it
        for blk in {x for b in bs.beams for x in b.table}:
            assert alloc.refcount(blk) == sum(b.table.count(blk) for b in bs.beams)
        assert bs.blocks_in_use() <= bs.blocks_unshared()
    bs.release()
    assert alloc.num_free == 200


def test_beam_search_all_continue_one_parent_shares_everything_but_the_last_block():
    B, W = 16, 4
    alloc = BlockAllocator(100, B)
    bs = BeamSearch(alloc, prompt_tokens=32, width=W)  # two full prompt blocks
    for _ in range(20):
        bs.step([0] * W)
    # 52 tokens: 3 full blocks + 4 tokens; the beams share the blocks beam 0
    # held, and each has its own last block
    tables = [b.table for b in bs.beams]
    assert all(t[:-1] == tables[0][:-1] for t in tables)
    assert len({t[-1] for t in tables}) == W
    assert bs.blocks_in_use() == len(tables[0]) - 1 + W


# ---------------------------------------------------------------------------
# automatic prefix caching (page "PagedAttention Analysis", section 4): blocks
# keyed by a hash of the whole prefix, shared through a global table
# ---------------------------------------------------------------------------

from pkv_inputs import PrefixCache  # noqa: E402


def test_prefix_keys_chain_the_whole_prefix():
    B = 16
    a = list(range(100))
    b = a[:32] + [7] * 68
    c = [999] + a[1:]
    ka, kb, kc = (PrefixCache.block_keys(t, B) for t in (a, b, c))
    assert len(ka) == 6  # full blocks only
    assert ka[:2] == kb[:2] and ka[2] != kb[2]
    assert all(x != y for x, y in zip(ka, kc))  # a change in block 0 changes every key


def test_prefix_cache_hits_misses_and_private_tails():
    B = 16
    pc = PrefixCache(BlockAllocator(64, B))
    sys_prompt = list(range(1000, 1064))  # 4 full blocks
    a, fa = pc.new_sequence(sys_prompt + list(range(40)))
    assert (pc.hits, pc.misses) == (0, 6) and fa == [0, 1, 2, 3, 4, 5, 6]
    b, fb = pc.new_sequence(sys_prompt + list(range(500, 540)))
    assert pc.hits == 4 and b.table[:4] == a.table[:4]
    assert fb == [4, 5, 6] and not set(b.table[4:]) & set(a.table)
    c, fc = pc.new_sequence(sys_prompt + list(range(40)))  # same tokens as a
    assert c.table[:6] == a.table[:6] and c.table[6] != a.table[6]  # the partial block is private
    assert fc == [6]
    assert pc.alloc.refcount(a.table[0]) == 3


def test_prefix_cache_survives_release_and_evicts_cleanly():
    B = 16
    alloc = BlockAllocator(12, B)
    pc = PrefixCache(alloc)
    toks = list(range(64))
    a, _ = pc.new_sequence(toks)
    a_table = list(a.table)
    pc.release(a)
    assert alloc.num_free == 12 and len(pc.table) == 4  # still cached
    b, fills = pc.new_sequence(toks)
    assert fills == [] and b.table == a_table  # all four blocks hit
    assert pc.hits == 4
    pc.release(b)
    # unrelated requests take the 8 empty blocks first, then evict cached
    # blocks, the prefix's last ones first; an evicted block leaves the table
    others = [pc.new_sequence([5000 + 100 * i + t for t in range(32)])[0] for i in range(5)]
    assert len(pc.table) == 2 + 10
    for k, blk in pc.table.items():
        assert pc.key_of[blk] == k
    for sq in others:
        pc.release(sq)
    c, fills = pc.new_sequence(toks)
    assert c.table[:2] == a_table[:2] and fills == [2, 3]  # blocks 0, 1 survived
    pc.release(c)
    assert alloc.num_free == 12
