"""The single-wave decode kernel (calls that fit one wave of CTAs) against the
fp64 oracle: cluster-merged partitions, warp-per-item short contexts, the fused
append, error reports, and agreement with the persistent kernel."""

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_387_b200 as pkv
from pkv_inputs import make_random_case
from tests.helpers import assert_close_to_oracle, gpu_decode, new_err, oracle_decode

pytestmark = pytest.mark.gpu
DEV = "cuda"
DT = {"f16": torch.float16, "bf16": torch.bfloat16}


@pytest.fixture
def dispatch():
    """Set a decode dispatch mode for one test and restore AUTO after it."""
    modes = []

    def set_mode(m):
        modes.append(pkv.set_decode_dispatch(m))

    yield set_mode
    pkv.set_decode_dispatch(pkv.DISPATCH_AUTO)


def ws_for(c, part):
    n = pkv.decode_workspace_bytes(c.num_seqs, c.num_heads, c.head_dim, c.max_context_len, part)
    return torch.full((max(n, 256),), 0xAB, dtype=torch.uint8, device=DEV)


def decode_ws(c, part, ws, err=None, fused=False):
    out = torch.empty_like(c.q)
    if fused:
        pkv.paged_attn_decode_append(out, c.q, c.k_new, c.v_new, c.k_pool, c.v_pool,
                                     c.block_tables, c.context_lens, c.scale,
                                     c.max_context_len, partition_size=part, workspace=ws,
                                     err=err)
    else:
        pkv.paged_attn_decode(out, c.q, c.k_pool, c.v_pool, c.block_tables, c.context_lens,
                              c.scale, c.max_context_len, partition_size=part, workspace=ws,
                              err=err)
    return out


def test_dispatch_setting_round_trips(dispatch):
    assert pkv.set_decode_dispatch(pkv.DISPATCH_PERSISTENT) == pkv.DISPATCH_AUTO
    assert pkv.set_decode_dispatch(pkv.DISPATCH_WAVE_CTA) == pkv.DISPATCH_PERSISTENT
    assert pkv.set_decode_dispatch(pkv.DISPATCH_WAVE_CTA8) == pkv.DISPATCH_WAVE_CTA
    assert pkv.set_decode_dispatch(pkv.DISPATCH_WAVE_CTA) == pkv.DISPATCH_WAVE_CTA8
    with pytest.raises(pkv.PkvError):
        pkv.set_decode_dispatch(7)
    assert pkv.set_decode_dispatch(pkv.DISPATCH_AUTO) == pkv.DISPATCH_WAVE_CTA


@pytest.mark.parametrize("lens,part", [([4096], pkv.PARTITION_AUTO), ([40, 3, 64], 0),
                                       ([300, 1000], 256)])
def test_wave_leaves_workspace_untouched(dispatch, lens, part):
    """A call that fits one wave runs without the plan and never writes the
    workspace; the persistent kernel writes its work list there."""
    c = make_random_case("ws", 32, 8, 128, 16, lens, torch.bfloat16, seed=4, device=DEV)
    ws = ws_for(c, part)
    out = decode_ws(c, part, ws)
    torch.cuda.synchronize()
    assert (ws == 0xAB).all()
    assert_close_to_oracle(out, oracle_decode(c), torch.bfloat16, "wave")
    dispatch(pkv.DISPATCH_PERSISTENT)
    out2 = decode_ws(c, part, ws)
    torch.cuda.synchronize()
    assert not (ws == 0xAB).all()
    assert_close_to_oracle(out2, oracle_decode(c), torch.bfloat16, "persistent")


# partitions per sequence from 2 to 16 (the largest cluster); the lengths end
# at every position of the last partition's tiles
@pytest.mark.parametrize("dt", ["f16", "bf16"])
@pytest.mark.parametrize("D,B", [(128, 16), (64, 32), (128, 8), (64, 24)])
@pytest.mark.parametrize("Hq,Hkv", [(8, 8), (32, 8), (8, 1), (6, 2)])
@pytest.mark.parametrize("nparts", [2, 3, 9, 16])
@pytest.mark.parametrize("mode", [pkv.DISPATCH_WAVE_CTA, pkv.DISPATCH_WAVE_CTA8])
def test_cluster_partitions_match_oracle(dt, D, B, Hq, Hkv, nparts, mode, dispatch):
    """4-warp CTAs, and 8-warp CTAs (at most one CTA per SM: these calls stay
    well below it)."""
    dispatch(mode)
    part = 128
    lens = [nparts * part, nparts * part - 17, (nparts - 1) * part + 1, 1, 0, 77]
    lens = lens[:max(1, min(len(lens), 120 // (Hkv * nparts)))]  # well inside one wave
    c = make_random_case("cl", Hq, Hkv, D, B, lens, DT[dt], seed=nparts + D + B + Hq,
                         device=DEV)
    ws = ws_for(c, part)
    err = new_err(DEV)
    got = decode_ws(c, part, ws, err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert (ws == 0xAB).all()  # it ran on the single-wave kernel
    assert_close_to_oracle(got, oracle_decode(c), DT[dt], f"{dt} D{D} B{B} G{Hq // Hkv} P{nparts}")


@pytest.mark.parametrize("dt", ["f16", "bf16"])
@pytest.mark.parametrize("D,B", [(128, 16), (64, 16), (128, 8), (64, 32)])
@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (32, 8), (8, 1), (14, 2)])
def test_warp_items_short_contexts(dt, D, B, Hq, Hkv):
    """Contexts of at most 64 tokens: one warp per (sequence, KV head), including
    a batch whose (sequence, KV head) count is not a multiple of 4 and lengths
    0 and 64."""
    rng = np.random.default_rng(D + B + Hq)
    lens = [0, 1, 64, 63, 16, 17] + [int(x) for x in rng.integers(0, 65, size=143)]
    c = make_random_case("warp", Hq, Hkv, D, B, lens, DT[dt], seed=Hq + B, device=DEV)
    ws = ws_for(c, pkv.PARTITION_AUTO)
    got = decode_ws(c, pkv.PARTITION_AUTO, ws)
    torch.cuda.synchronize()
    assert (ws == 0xAB).all()
    assert (got[0] == 0).all()
    assert_close_to_oracle(got, oracle_decode(c), DT[dt], f"warp {dt} D{D} B{B} G{Hq // Hkv}")


@pytest.mark.parametrize("D,B", [(128, 16), (64, 8)])
def test_warp_items_forced_on_long_contexts(D, B, dispatch):
    """The warp form on contexts of up to 80 tiles: the block ids of a warp's
    tiles are fetched 32 at a time, so this crosses two refills."""
    dispatch(pkv.DISPATCH_WAVE_WARP)
    c = make_random_case("warp_long", 16, 4, D, B, [1280, 513, 1, 999, 512, 0, 31], torch.bfloat16,
                         seed=B, device=DEV)
    ws = ws_for(c, 0)
    got = decode_ws(c, 0, ws)
    torch.cuda.synchronize()
    assert (ws == 0xAB).all()
    assert_close_to_oracle(got, oracle_decode(c), torch.bfloat16, f"forced warp D{D} B{B}")


@pytest.mark.parametrize("dt", ["f16", "bf16"])
@pytest.mark.parametrize("lens", [[4096], [8192], [3000, 1, 7001], [20000, 5, 900, 16, 333],
                                  [4096] * 4])
def test_auto_partition_single_wave(dt, lens):
    """PARTITION_AUTO on small batches of long contexts: the single-wave kernel
    chooses up to 16 partitions per sequence."""
    c = make_random_case("auto_w", 32, 8, 128, 16, lens, DT[dt], seed=len(lens), device=DEV)
    ws = ws_for(c, pkv.PARTITION_AUTO)
    got = decode_ws(c, pkv.PARTITION_AUTO, ws)
    torch.cuda.synchronize()
    assert (ws == 0xAB).all()
    assert_close_to_oracle(got, oracle_decode(c), DT[dt], f"auto {dt} {lens}")


@pytest.mark.parametrize("dt", ["f16", "bf16"])
@pytest.mark.parametrize("mode", ["cta", "cta8", "warp"])
@pytest.mark.parametrize("D,B", [(128, 16), (64, 32), (128, 8)])
def test_fused_append_single_wave(dt, mode, D, B, dispatch):
    """The fused append on the single-wave kernel: the pool after the call
    equals the oracle's append bit for bit, and the output its decode."""
    if mode == "cta":
        dispatch(pkv.DISPATCH_WAVE_CTA)
        lens, part = [1, 2, 15, 16, 17, 31, 33, 100, 511, 512, 513, 1000], 256
    elif mode == "cta8":  # 7 x 4 KV heads x 4 partitions: one 8-warp CTA per SM at most
        dispatch(pkv.DISPATCH_WAVE_CTA8)
        lens, part = [1, 2, 17, 33, 511, 513, 1000], 256
    else:
        lens, part = [1, 2, 8, 9, 15, 16, 17, 31, 32, 33, 48, 63, 64], 0
    c = make_random_case("fw", 16, 4, D, B, lens, DT[dt], seed=D + B, device=DEV,
                         with_append=True)
    kc, vc = c.k_pool.cpu(), c.v_pool.cpu()
    oracle.cache_append(kc, vc, c.k_new.cpu(), c.v_new.cpu(), c.slot_mapping.cpu())
    ref = oracle.paged_decode(c.q.cpu(), kc, vc, c.block_tables.cpu(), c.context_lens.cpu(),
                              c.scale)
    ws = ws_for(c, part)
    err = new_err(DEV)
    out = decode_ws(c, part, ws, err=err, fused=True)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert (ws == 0xAB).all()
    assert torch.equal(c.k_pool.cpu().view(torch.int16), kc.view(torch.int16))
    assert torch.equal(c.v_pool.cpu().view(torch.int16), vc.view(torch.int16))
    assert_close_to_oracle(out, ref, DT[dt], f"fused {mode} {dt} D{D} B{B}")


@pytest.mark.parametrize("mode", [pkv.DISPATCH_WAVE_CTA, pkv.DISPATCH_WAVE_CTA8,
                                  pkv.DISPATCH_WAVE_WARP])
@pytest.mark.parametrize("B,entry", [(16, 1), (8, 1), (8, 2)])
def test_bad_block_id_reports_and_masks(mode, B, entry, dispatch):
    dispatch(mode)
    c = make_random_case("bad_w", 4, 4, 128, B, [40, 20], torch.bfloat16, seed=9, device=DEV)
    bt = c.block_tables.clone()
    bt[0, entry] = c.num_blocks + 5
    c.block_tables = bt
    err = new_err(DEV)
    got = gpu_decode(c, partition_size=0, err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 1  # PKV_DEV_BAD_BLOCK
    # the masked tile's tokens drop out of sequence 0; sequence 1 is unaffected
    assert_close_to_oracle(got[1:], oracle_decode(c, seqs=[1]), torch.bfloat16, "bad id, seq 1")
    assert not torch.isnan(got).any()


@pytest.mark.parametrize("mode", [pkv.DISPATCH_WAVE_CTA, pkv.DISPATCH_WAVE_CTA8,
                                  pkv.DISPATCH_WAVE_WARP])
def test_context_len_above_max_reports(mode, dispatch):
    dispatch(mode)
    c = make_random_case("clamp_w", 8, 2, 64, 16, [30, 50], torch.float16, seed=2, device=DEV)
    err = new_err(DEV)
    got = gpu_decode(c, partition_size=0, err=err, max_context_len=40)
    torch.cuda.synchronize()
    assert int(err.item()) == 4  # PKV_DEV_CONTEXT_LEN
    assert_close_to_oracle(got[:1], oracle_decode(c, seqs=[0]), torch.float16, "unclamped seq")


@pytest.mark.parametrize("lens,part", [([700, 5, 1500, 64], 256), ([4096], pkv.PARTITION_AUTO),
                                       ([60] * 40, 0)])
def test_wave_and_persistent_agree(lens, part, dispatch):
    c = make_random_case("agree", 32, 8, 128, 16, lens, torch.bfloat16, seed=len(lens),
                         device=DEV)
    wave = gpu_decode(c, partition_size=part)
    dispatch(pkv.DISPATCH_PERSISTENT)
    pers = gpu_decode(c, partition_size=part)
    ref = oracle_decode(c)
    assert_close_to_oracle(wave, ref, torch.bfloat16, "wave")
    assert_close_to_oracle(pers, ref, torch.bfloat16, "persistent")
    d = (wave.float() - pers.float()).abs().max().item()
    assert d <= 2e-2, d


def test_back_to_back_single_wave_calls_in_a_graph():
    """Single-wave calls chained by programmatic launch inside a CUDA graph:
    every replay gives the same bits as an eager call."""
    c = make_random_case("graph_w", 32, 8, 128, 16, [4096, 100], torch.bfloat16, seed=5,
                         device=DEV)
    ref = gpu_decode(c, partition_size=pkv.PARTITION_AUTO)
    outs = [torch.empty_like(c.q) for _ in range(4)]
    mcl = c.max_context_len  # (a device read: not inside the capture)
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for o in outs:
            pkv.paged_attn_decode(o, c.q, c.k_pool, c.v_pool, c.block_tables, c.context_lens,
                                  c.scale, mcl, partition_size=pkv.PARTITION_AUTO, stream=s)
    for _ in range(3):
        for o in outs:
            o.zero_()
        g.replay()
        torch.cuda.synchronize()
        for o in outs:
            assert torch.equal(o, ref)


@pytest.mark.parametrize("dt", ["f16", "bf16"])
@pytest.mark.parametrize("lens,fused", [([65536], False), ([65536], True), ([100000], False),
                                        ([131072], False)])
def test_long_contexts_split_over_clusters(dt, lens, fused):
    """A few very long contexts under PARTITION_AUTO: several clusters per
    (sequence, KV head) each merge their partitions into a workspace slot,
    and a merge launch combines the slots. The plan's words at the start of
    the workspace stay untouched (no persistent kernel ran); the slots do not."""
    c = make_random_case("split_w", 32, 8, 128, 16, lens, DT[dt], seed=len(lens) + lens[0] % 7,
                         device=DEV, with_append=fused)
    ws = ws_for(c, pkv.PARTITION_AUTO)
    err = new_err(DEV)
    if fused:
        kc, vc = c.k_pool.cpu(), c.v_pool.cpu()
        oracle.cache_append(kc, vc, c.k_new.cpu(), c.v_new.cpu(), c.slot_mapping.cpu())
        ref = oracle.paged_decode(c.q.cpu(), kc, vc, c.block_tables.cpu(), c.context_lens.cpu(),
                                  c.scale)
    else:
        ref = oracle_decode(c)
    got = decode_ws(c, pkv.PARTITION_AUTO, ws, err=err, fused=fused)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert (ws[:256] == 0xAB).all()
    assert not (ws == 0xAB).all()
    if fused:
        assert torch.equal(c.k_pool.cpu().view(torch.int16), kc.view(torch.int16))
    assert_close_to_oracle(got, ref, DT[dt], f"split clusters {dt} {lens}")


@pytest.mark.parametrize("Hq,Hkv,D,B,dt", [(8, 1, 64, 8, "f16"), (16, 2, 128, 32, "bf16"),
                                           (6, 2, 64, 16, "bf16")])
def test_split_form_shapes(Hq, Hkv, D, B, dt):
    """The split form over head dims, block sizes (8: two blocks per tile) and
    group sizes, with up to 32 clusters per KV head; fused append included."""
    c = make_random_case("split_shapes", Hq, Hkv, D, B, [65536], DT[dt], seed=Hq + D + B,
                         device=DEV, with_append=True)
    kc, vc = c.k_pool.cpu(), c.v_pool.cpu()
    oracle.cache_append(kc, vc, c.k_new.cpu(), c.v_new.cpu(), c.slot_mapping.cpu())
    ref = oracle.paged_decode(c.q.cpu(), kc, vc, c.block_tables.cpu(), c.context_lens.cpu(),
                              c.scale)
    ws = ws_for(c, pkv.PARTITION_AUTO)
    err = new_err(DEV)
    got = decode_ws(c, pkv.PARTITION_AUTO, ws, err=err, fused=True)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert (ws[:256] == 0xAB).all()
    assert not (ws == 0xAB).all()
    assert torch.equal(c.v_pool.cpu().view(torch.int16), vc.view(torch.int16))
    assert_close_to_oracle(got, ref, DT[dt], f"split D{D} B{B} G{Hq // Hkv}")
