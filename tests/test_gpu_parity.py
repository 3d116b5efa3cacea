"""Parity of the CUDA path (through the C ABI) against the fp64 CPU oracle."""


import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_387_b200 as pkv
from pkv_inputs import make_case, make_random_case, make_shared_prefix_case
from tests.helpers import assert_close_to_oracle, gpu_decode, new_err, oracle_decode

pytestmark = pytest.mark.gpu

DEV = "cuda"
DT = {"f16": torch.float16, "bf16": torch.bfloat16, "f32": torch.float32}


@pytest.fixture(autouse=True, params=["auto", "persistent"])
def _dispatch(request):
    """Every test runs under the default kernel selection (small calls take the
    single-wave kernel) and with the persistent kernel forced."""
    if request.param == "persistent":
        pkv.set_decode_dispatch(pkv.DISPATCH_PERSISTENT)
    yield
    pkv.set_decode_dispatch(pkv.DISPATCH_AUTO)


# ---------------------------------------------------------------------------
# decode: small cases spanning several tiles and a ragged tail
# ---------------------------------------------------------------------------

EDGE_LENS = [1, 15, 16, 17, 31, 37, 63, 64, 65, 200, 513, 1100]


@pytest.mark.parametrize("dt", ["f16", "bf16"])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("B", [8, 16, 24, 32])  # 8, 24: a tile spans two blocks
@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (8, 2), (8, 1), (16, 2)])
@pytest.mark.parametrize("part", [0, 64, 512])
def test_decode_16bit_matches_oracle(dt, D, B, Hq, Hkv, part):
    c = make_random_case("edge", Hq, Hkv, D, B, EDGE_LENS, DT[dt], seed=100 + D + B + Hq,
                         device=DEV, pool_blocks=None)
    got = gpu_decode(c, partition_size=part)
    assert_close_to_oracle(got, oracle_decode(c), DT[dt], f"{dt} D{D} B{B} G{Hq // Hkv} p{part}")


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("B", [1, 7, 16, 32])
@pytest.mark.parametrize("part", [0, 16, 512])
def test_decode_f32_matches_oracle(D, B, part):
    c = make_random_case("edge32", 4, 2, D, B, EDGE_LENS, torch.float32, seed=7 + B, device=DEV)
    got = gpu_decode(c, partition_size=part)
    assert_close_to_oracle(got, oracle_decode(c), torch.float32, f"f32 D{D} B{B} p{part}")


def test_tiny_fp32_workload():
    c = make_case("tiny_f32", device=DEV)
    for part in (0, 16, 512):
        got = gpu_decode(c, partition_size=part)
        assert_close_to_oracle(got, oracle_decode(c), torch.float32, f"tiny p{part}")


def test_block_size_64_and_256():
    for B in (64, 256):
        c = make_random_case("bigblock", 8, 2, 128, B, [1, 300, 700, 64, 65], torch.bfloat16,
                             seed=B, device=DEV)
        assert_close_to_oracle(gpu_decode(c), oracle_decode(c), torch.bfloat16, f"B{B}")


@pytest.mark.parametrize("dt", ["f16", "bf16", "f32"])
@pytest.mark.parametrize("lens", [[4096], [3000, 1, 7001], [20000, 5, 900, 16, 333]])
def test_auto_partition_small_batches(dt, lens):
    """PARTITION_AUTO splits a small batch of long contexts into short
    partitions (256 tokens for one 4096-token sequence of 8 heads; 26
    partitions, two merge levels, for the 20000-token one); the result must
    still match the oracle."""
    D = 64 if dt == "f32" else 128
    c = make_random_case("auto", 8, 2, D, 16, lens, DT[dt], seed=len(lens) + D, device=DEV)
    part = pkv.resolve_partition(c.num_seqs, c.num_heads, c.max_context_len)
    assert 256 <= part < max(lens)  # the contexts are split
    got = gpu_decode(c, partition_size=pkv.PARTITION_AUTO)
    assert_close_to_oracle(got, oracle_decode(c), DT[dt], f"{dt} auto partition {part}")


def test_placement_invariance_and_contiguous_equality():
    kw = dict(name="perm", num_heads=8, num_kv_heads=2, head_dim=128, block_size=16,
              context_lens=[3, 77, 300, 1030], dtype=torch.bfloat16, seed=55, device=DEV,
              pool_blocks=120)
    outs = []
    for placement in ("identity", "shuffle"):
        c = make_random_case(placement=placement, **kw)
        outs.append(gpu_decode(c, partition_size=512))
    for seed_shift in (1, 2):
        c = make_random_case(placement="shuffle", **kw)
        # same tokens, another physical placement: permute blocks and remap tables
        perm = torch.as_tensor(np.random.default_rng(seed_shift).permutation(c.num_blocks),
                               device=DEV)
        kp = torch.empty_like(c.k_pool)
        vp = torch.empty_like(c.v_pool)
        kp[perm] = c.k_pool
        vp[perm] = c.v_pool
        bt = torch.where(c.block_tables >= 0, perm[c.block_tables.long().clamp(min=0)].int(),
                         c.block_tables)
        out = torch.empty_like(c.q)
        pkv.paged_attn_decode(out, c.q, kp, vp, bt.contiguous(), c.context_lens, c.scale,
                              c.max_context_len, partition_size=512)
        outs.append(out)
    for o in outs[1:]:
        assert torch.equal(o, outs[0])  # same arithmetic order: identical bits


@pytest.mark.parametrize("B", [16, 8])
def test_zero_length_and_tail_poison(B):
    c = make_random_case("zero", 4, 2, 128, B, [0, 5, 16, 0, 33], torch.float16, seed=3,
                         device=DEV, pool_blocks=160 // B)
    got = gpu_decode(c, partition_size=16)
    assert torch.isnan(c.k_pool).any()  # poisoned slots exist
    assert (got[0] == 0).all() and (got[3] == 0).all()
    assert_close_to_oracle(got, oracle_decode(c), torch.float16, "zero/poison")


@pytest.mark.parametrize("B,entry", [(16, 1), (8, 1), (8, 2)])
def test_bad_block_id_reports_and_masks(B, entry):
    # with B = 8, entry 1 is the second unit of tile 0 and entry 2 the first of tile 1
    c = make_random_case("bad", 4, 4, 128, B, [40, 20], torch.bfloat16, seed=9, device=DEV)
    bt = c.block_tables.clone()
    bt[0, entry] = c.num_blocks + 5
    c.block_tables = bt
    err = new_err(DEV)
    got = gpu_decode(c, err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 1
    assert not torch.isnan(got.float()).any()
    # sequence 1 is untouched by the bad entry of sequence 0
    ref1 = oracle_decode(c, seqs=[1])
    assert_close_to_oracle(got[1:], ref1, torch.bfloat16, "seq 1")


def test_context_len_above_max_reports():
    c = make_random_case("clamp", 4, 4, 64, 16, [100, 20], torch.float16, seed=2, device=DEV)
    err = new_err(DEV)
    gpu_decode(c, err=err, max_context_len=64)
    torch.cuda.synchronize()
    assert int(err.item()) == 4


def test_host_checked_errors():
    c = make_random_case("args", 4, 4, 128, 16, [20], torch.bfloat16, seed=2, device=DEV)
    with pytest.raises(pkv.PkvError) as e:
        gpu_decode(c, partition_size=24)
    assert e.value.status == pkv.PKV_EINVAL
    c12 = make_random_case("b12", 4, 4, 128, 12, [20], torch.bfloat16, seed=2, device=DEV)
    with pytest.raises(pkv.PkvError) as e:  # 16-bit block sizes are multiples of 8
        gpu_decode(c12)
    assert e.value.status == pkv.PKV_EUNSUPPORTED


# ---------------------------------------------------------------------------
# append and block copy: bit-exact over the whole pool
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("dt", ["f16", "bf16", "f32"])
def test_append_bit_exact(dt):
    c = make_random_case("app", 8, 4, 128, 16, [5, 16, 17, 40, 1], DT[dt], seed=12, device=DEV,
                         with_append=True, pool_blocks=20)
    kc, vc = c.k_pool.cpu().clone(), c.v_pool.cpu().clone()
    sm = c.slot_mapping.clone()
    sm[1] = -1  # skipped token
    pkv.kv_cache_append(c.k_pool, c.v_pool, c.k_new, c.v_new, sm)
    oracle.cache_append(kc, vc, c.k_new.cpu(), c.v_new.cpu(), sm.cpu())
    torch.cuda.synchronize()
    ik = torch.int32 if dt == "f32" else torch.int16
    assert torch.equal(c.k_pool.cpu().view(ik), kc.view(ik))
    assert torch.equal(c.v_pool.cpu().view(ik), vc.view(ik))


def test_append_bad_slot_reports():
    c = make_random_case("app", 4, 4, 64, 16, [5, 9], torch.float16, seed=1, device=DEV,
                         with_append=True)
    sm = c.slot_mapping.clone()
    sm[0] = c.num_blocks * 16
    err = new_err(DEV)
    before = c.k_pool.clone()
    pkv.kv_cache_append(c.k_pool, c.v_pool, c.k_new, c.v_new, sm, err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 2
    changed = (c.k_pool.view(torch.int16) != before.view(torch.int16)).any(dim=(1, 2, 3))
    assert int(changed.sum()) == 1  # only the valid token's block


@pytest.mark.parametrize("dt", ["f16", "bf16", "f32"])
def test_block_copy_bit_exact(dt):
    c = make_random_case("cp", 4, 3, 64, 32, [100, 70], DT[dt], seed=4, device=DEV,
                         pool_blocks=16)
    pairs = torch.tensor([[0, 9], [3, 12], [5, 15]], dtype=torch.int32)
    kc, vc = c.k_pool.cpu().clone(), c.v_pool.cpu().clone()
    pkv.kv_block_copy(c.k_pool, c.v_pool, pairs.to(DEV))
    oracle.block_copy(kc, vc, pairs)
    torch.cuda.synchronize()
    ik = torch.int32 if dt == "f32" else torch.int16
    assert torch.equal(c.k_pool.cpu().view(ik), kc.view(ik))
    assert torch.equal(c.v_pool.cpu().view(ik), vc.view(ik))


def test_block_copy_bad_pair_reports():
    c = make_random_case("cp", 2, 2, 64, 16, [20], torch.float16, seed=4, device=DEV,
                         pool_blocks=4)
    err = new_err(DEV)
    pkv.kv_block_copy(c.k_pool, c.v_pool, torch.tensor([[0, 7]], dtype=torch.int32,
                                                       device=DEV), err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 3


# ---------------------------------------------------------------------------
# the five workloads at full size
# ---------------------------------------------------------------------------

def test_workload_opt13b_append_then_decode():
    c = make_case("opt13b_mha_b64", device=DEV)           # append precedes decode
    kc, vc = c.k_pool.cpu(), c.v_pool.cpu()
    pkv.kv_cache_append(c.k_pool, c.v_pool, c.k_new, c.v_new, c.slot_mapping)
    oracle.cache_append(kc, vc, c.k_new.cpu(), c.v_new.cpu(), c.slot_mapping.cpu())
    torch.cuda.synchronize()
    assert torch.equal(c.k_pool.cpu().view(torch.int16), kc.view(torch.int16))
    got = gpu_decode(c)
    ref = oracle.paged_decode(c.q.cpu(), kc, vc, c.block_tables.cpu(), c.context_lens.cpu(),
                              c.scale)
    assert_close_to_oracle(got, ref, torch.float16, "opt13b")


def test_workload_llama8b_gqa_sampled():
    c = make_case("llama8b_gqa_b256", device=DEV)
    got = gpu_decode(c)
    lens = c.context_lens.cpu().numpy()
    order = np.argsort(lens)
    seqs = sorted(set(order[:8].tolist() + order[-8:].tolist() +
                      np.random.default_rng(0).choice(len(lens), 24, replace=False).tolist()))
    ref = oracle_decode(c, seqs=seqs)
    assert_close_to_oracle(got[torch.as_tensor(seqs, device=DEV)], ref, torch.bfloat16,
                           "llama8b sampled")


def test_workload_long_split_sampled():
    c = make_case("long_split_b8", device=DEV)
    got = gpu_decode(c)
    lens = c.context_lens.cpu().numpy()
    seqs = [int(np.argmin(lens)), int(np.argmax(lens))]
    ref = oracle_decode(c, seqs=seqs)
    assert_close_to_oracle(got[torch.as_tensor(seqs, device=DEV)], ref, torch.bfloat16,
                           "long split sampled")


def test_workload_shared_prefix_cow_pipeline():
    sp = make_shared_prefix_case(device=DEV, decode_steps=64)
    kc, vc = sp.k_pool.cpu(), sp.v_pool.cpu()
    pkv.kv_block_copy(sp.k_pool, sp.v_pool, sp.cow_pairs)
    oracle.block_copy(kc, vc, sp.cow_pairs.cpu())
    checked = 0
    for k, st in enumerate(sp.steps):
        q, kn, vn = sp.step_tokens(k)
        pkv.kv_cache_append(sp.k_pool, sp.v_pool, kn, vn, st["slot_mapping"])
        oracle.cache_append(kc, vc, kn.cpu(), vn.cpu(), st["slot_mapping"].cpu())
        out = torch.empty_like(q)
        pkv.paged_attn_decode(out, q, sp.k_pool, sp.v_pool, st["block_tables"],
                              st["context_lens"], sp.scale, int(st["context_lens"].max()),
                              partition_size=512)
        if k in (0, 1, 31, 63):
            ref = oracle.paged_decode(q.cpu(), kc, vc, st["block_tables"].cpu(),
                                      st["context_lens"].cpu(), sp.scale)
            assert_close_to_oracle(out, ref, torch.float16, f"shared prefix step {k}")
            checked += 1
    torch.cuda.synchronize()
    assert checked == 4
    assert torch.equal(sp.k_pool.cpu().view(torch.int16), kc.view(torch.int16))
    assert torch.equal(sp.v_pool.cpu().view(torch.int16), vc.view(torch.int16))


@pytest.mark.parametrize("dt", ["f16", "bf16"])
@pytest.mark.parametrize("seed", range(6))
def test_decode_accuracy_short_contexts_with_cancellation(dt, seed):
    # Short contexts: a few weights, value rows that often nearly cancel, so
    # the output is small and the absolute bound 2e-3 is what matters.
    lens = [2, 3, 2, 4, 5, 2, 3, 8] * 8
    c = make_random_case("short", 32, 8, 128, 16, lens, DT[dt], seed=1000 + seed, device=DEV)
    for part in (0, 16):
        got = gpu_decode(c, partition_size=part)
        assert_close_to_oracle(got, oracle_decode(c), DT[dt], f"short {dt} s{seed} p{part}")


@pytest.mark.parametrize("dt,B,part", [(torch.bfloat16, 16, 0), (torch.float16, 8, 32)])
def test_many_short_sequences(dt, B, part):
    """Thousands of sequences (the plan takes them in many rounds; contexts of 0
    to 80 tokens; with 32-token partitions many are split), every output
    checked against the oracle."""
    lens = np.random.default_rng(13).integers(0, 81, size=3000).tolist()
    c = make_random_case("many", 8, 2, 64, B, lens, dt, seed=29, device=DEV)
    err = new_err(DEV)
    got = gpu_decode(c, partition_size=part, err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert_close_to_oracle(got, oracle_decode(c), dt, f"3000 seqs B{B} p{part}")


def test_max_group_and_block_size():
    """The largest supported group (8 query heads per KV head) with the largest
    block size (256 tokens), contexts spanning several blocks and partitions."""
    c = make_random_case("maxgb", 32, 4, 128, 256, [1, 255, 256, 257, 1500, 3000], torch.bfloat16,
                         seed=31, device=DEV)
    for part in (0, 256, 1024):
        assert_close_to_oracle(gpu_decode(c, partition_size=part), oracle_decode(c),
                               torch.bfloat16, f"G8 B256 p{part}")


@pytest.mark.parametrize("fused", [False, True])
def test_back_to_back_calls_with_changing_batches(fused):
    """Consecutive calls overlap: a call's plan builds its work list while the
    previous call is still running, and stores it once that call is done.
    Batches of different sizes and lengths alternate on one workspace; every
    output must equal the batch's output from a call made alone."""
    lens_sets = [[5, 300, 1200, 40], [2100, 17, 64, 700, 33, 1000, 1], [129] * 20]
    cases = [make_random_case(f"b2b{i}", 8, 2, 128, 16, lens, torch.bfloat16, seed=40 + i,
                              device=DEV, with_append=fused)
             for i, lens in enumerate(lens_sets)]
    part = 64

    def call(c, out, ws=None):
        if fused:  # appending the same token again leaves the pool unchanged
            pkv.paged_attn_decode_append(out, c.q, c.k_new, c.v_new, c.k_pool, c.v_pool,
                                         c.block_tables, c.context_lens, c.scale,
                                         c.max_context_len, partition_size=part, workspace=ws)
        else:
            pkv.paged_attn_decode(out, c.q, c.k_pool, c.v_pool, c.block_tables, c.context_lens,
                                  c.scale, c.max_context_len, partition_size=part, workspace=ws)

    refs = []
    for c in cases:
        o = torch.empty_like(c.q)
        call(c, o)
        torch.cuda.synchronize()
        refs.append(o)
    need = max(pkv.decode_workspace_bytes(c.num_seqs, c.num_heads, c.head_dim,
                                          c.max_context_len, part) for c in cases)
    ws = torch.empty(need, dtype=torch.uint8, device=DEV)
    outs = []
    for i in range(45):
        c = cases[i % 3]
        o = torch.empty_like(c.q)
        call(c, o, ws)
        outs.append((i % 3, o))
    torch.cuda.synchronize()
    for k, o in outs:
        assert torch.equal(o.view(torch.int16), refs[k].view(torch.int16)), f"batch {k}"


@pytest.mark.parametrize("S", [1, 2, 31, 32, 33, 64])
@pytest.mark.parametrize("part", [0, 64])
def test_small_batches_plan_paths(S, part):
    """Up to 32 sequences without shared-prefix groups are planned by one warp,
    larger batches by the whole plan block: both must give the same work (every
    partition of every sequence, empty sequences included)."""
    rng = np.random.default_rng(S + part)
    lens = rng.integers(0, 300, size=S).tolist()
    lens[0] = 0
    if S > 2:
        lens[1] = 257  # several 64-token partitions
    c = make_random_case("smallS", 16, 4, 128, 16, lens, torch.bfloat16, seed=S, device=DEV)
    err = new_err(DEV)
    got = gpu_decode(c, partition_size=part, err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert (got[0] == 0).all()
    assert_close_to_oracle(got, oracle_decode(c), torch.bfloat16, f"S{S} p{part}")
