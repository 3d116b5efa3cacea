"""kv_block_swap (device pool <-> swap space in pinned host memory) against the
oracle: the swap space after a swap-out, and the device pool after a swap-in,
must equal the oracle's block swap bit for bit, and a decode after the round
trip (into other physical blocks) must give the same output as before."""

import pytest
import torch

import oracle
import paged_kv_cache_387_b200 as pkv
from pkv_inputs import BlockAllocator, SwapSpace, make_random_case
from tests.helpers import assert_close_to_oracle, gpu_decode, new_err, oracle_decode

pytestmark = pytest.mark.gpu
DEV = "cuda"
DT = {"f16": torch.float16, "bf16": torch.bfloat16, "f32": torch.float32}
BITS = {torch.float16: torch.int16, torch.bfloat16: torch.int16, torch.float32: torch.int32}
LENS = [40, 1, 300, 17, 129, 64, 1000, 5]


def adopt_case(c):
    """A GPU allocator holding the case's block tables."""
    P, B = c.num_blocks, c.block_size
    gpu = BlockAllocator(P, B)
    lens = c.context_lens.cpu().tolist()
    bt = c.block_tables.cpu().numpy()
    seqs = [gpu.adopt(bt[s, :-(-L // B)].tolist(), L) for s, L in enumerate(lens)]
    return gpu, seqs


def pairs_of(moves, device=DEV, pin=False):
    a = torch.tensor([[m.src, m.dst] for m in moves], dtype=torch.int32)
    return a.pin_memory() if pin else a.to(device)


def set_tables(c, seqs):
    bt = c.block_tables.cpu().clone()
    for s, sq in enumerate(seqs):
        if not sq.on_host:
            bt[s, :len(sq.table)] = torch.tensor(sq.table, dtype=torch.int32)
    c.block_tables = bt.to(DEV)


@pytest.mark.parametrize("dt", ["f16", "bf16", "f32"])
@pytest.mark.parametrize("B", [16, 8])
@pytest.mark.parametrize("pin_pairs", [False, True])
def test_swap_round_trip(dt, B, pin_pairs):
    if dt == "f32" and B == 8:
        pytest.skip("one block size is enough for the fp32 decode here")
    c = make_random_case("swap", 8, 2, 128, B, LENS, DT[dt], seed=21 + B, device=DEV,
                         pool_blocks=2 * sum(-(-L // B) for L in LENS) + 3)
    out_before = gpu_decode(c, partition_size=512)
    gpu, seqs = adopt_case(c)
    sw = SwapSpace(gpu)
    Pc = sw.cpu.num_blocks
    shape = (Pc,) + tuple(c.k_pool.shape[1:])
    hk = torch.full(shape, float("nan"), dtype=c.k_pool.dtype).pin_memory()
    hv = torch.full(shape, float("nan"), dtype=c.k_pool.dtype).pin_memory()
    ek, ev = hk.clone(), hv.clone()  # the oracle's swap space
    dk, dv = c.k_pool.cpu(), c.v_pool.cpu()  # the oracle's device pools
    err = new_err(DEV)
    group = [seqs[0], seqs[2], seqs[6]]

    # swap-out: device -> host
    out_moves = sw.swap_out(group)
    pkv.kv_block_swap(hk, hv, c.k_pool, c.v_pool, pairs_of(out_moves, pin=pin_pairs), err=err)
    torch.cuda.synchronize()
    oracle.block_swap(ek, ev, dk, dv, pairs_of(out_moves, pin=False).cpu().numpy())
    assert torch.equal(hk.view(BITS[c.k_pool.dtype]), ek.view(BITS[c.k_pool.dtype]))
    assert torch.equal(hv.view(BITS[c.k_pool.dtype]), ev.view(BITS[c.k_pool.dtype]))

    # the freed GPU blocks are reused by another sequence and overwritten
    squatter = gpu.new_sequence(len(out_moves) * B)
    idx = torch.tensor(squatter.table, device=DEV, dtype=torch.long)
    c.k_pool[idx] = float("nan")
    c.v_pool[idx] = float("nan")
    dk[idx.cpu()] = float("nan")
    dv[idx.cpu()] = float("nan")

    # swap-in: host -> device, into other physical blocks
    in_moves = sw.swap_in(group)
    assert not set(m.dst for m in in_moves) & set(squatter.table)
    pkv.kv_block_swap(c.k_pool, c.v_pool, hk, hv, pairs_of(in_moves, pin=pin_pairs), err=err)
    torch.cuda.synchronize()
    oracle.block_swap(dk, dv, ek, ev, pairs_of(in_moves, pin=False).cpu().numpy())
    assert int(err.item()) == 0
    assert torch.equal(c.k_pool.cpu().view(BITS[c.k_pool.dtype]), dk.view(BITS[c.k_pool.dtype]))
    assert torch.equal(c.v_pool.cpu().view(BITS[c.k_pool.dtype]), dv.view(BITS[c.k_pool.dtype]))

    set_tables(c, seqs)
    out_after = gpu_decode(c, partition_size=512)
    # the same tokens in other blocks: the decode is bit-identical
    assert torch.equal(out_after.view(BITS[c.k_pool.dtype]), out_before.view(BITS[c.k_pool.dtype]))
    assert_close_to_oracle(out_after, oracle_decode(c), c.k_pool.dtype, f"after swap {dt} B{B}")


def test_swap_bad_pair_reports_and_skips():
    c = make_random_case("swapbad", 4, 4, 64, 16, [20, 40], torch.float16, seed=5, device=DEV)
    P = c.num_blocks
    shape = (2,) + tuple(c.k_pool.shape[1:])
    hk = torch.zeros(shape, dtype=torch.float16).pin_memory()
    hv = torch.zeros(shape, dtype=torch.float16).pin_memory()
    err = new_err(DEV)
    pairs = torch.tensor([[0, 0], [P, 1], [1, 2]], dtype=torch.int32, device=DEV)
    pkv.kv_block_swap(hk, hv, c.k_pool, c.v_pool, pairs, err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 3
    assert torch.equal(hk[0].view(torch.int16), c.k_pool[0].cpu().view(torch.int16))
    assert (hk[1] == 0).all()  # the bad pairs were skipped
