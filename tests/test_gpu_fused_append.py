"""paged_attn_decode_append (cache-append fused into decode) against the oracle:
the pool after the call must equal the oracle's append bit for bit, and the
output must match the oracle's decode over the appended cache."""

import pytest
import torch

import oracle
import paged_kv_cache_387_b200 as pkv
from pkv_inputs import make_case, make_random_case, make_shared_prefix_case
from tests.helpers import assert_close_to_oracle

pytestmark = pytest.mark.gpu
DEV = "cuda"
DT = {"f16": torch.float16, "bf16": torch.bfloat16}


@pytest.fixture(autouse=True, params=["auto", "persistent"])
def _dispatch(request):
    """Every test runs under the default kernel selection (small calls take the
    single-wave kernel) and with the persistent kernel forced."""
    if request.param == "persistent":
        pkv.set_decode_dispatch(pkv.DISPATCH_PERSISTENT)
    yield
    pkv.set_decode_dispatch(pkv.DISPATCH_AUTO)


def fused_vs_oracle(c, part, what):
    kc, vc = c.k_pool.cpu(), c.v_pool.cpu()
    oracle.cache_append(kc, vc, c.k_new.cpu(), c.v_new.cpu(), c.slot_mapping.cpu())
    ref = oracle.paged_decode(c.q.cpu(), kc, vc, c.block_tables.cpu(), c.context_lens.cpu(),
                              c.scale)
    out = torch.empty_like(c.q)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    pkv.paged_attn_decode_append(out, c.q, c.k_new, c.v_new, c.k_pool, c.v_pool,
                                 c.block_tables, c.context_lens, c.scale, c.max_context_len,
                                 partition_size=part, err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert torch.equal(c.k_pool.cpu().view(torch.int16), kc.view(torch.int16)), what
    assert torch.equal(c.v_pool.cpu().view(torch.int16), vc.view(torch.int16)), what
    assert_close_to_oracle(out, ref, c.q.dtype, what)


# every position of the newest token inside its tile and block, tile edges included
LENS = [1, 2, 15, 16, 17, 31, 32, 33, 48, 100, 511, 512, 513, 1000, 2049]


@pytest.mark.parametrize("dt", ["f16", "bf16"])
@pytest.mark.parametrize("D,B", [(128, 16), (64, 32), (128, 64), (128, 8), (64, 24)])
@pytest.mark.parametrize("Hq,Hkv", [(8, 8), (16, 4), (8, 1)])
@pytest.mark.parametrize("part", [0, 512, 2048])
def test_fused_append_decode_matches_append_then_decode(dt, D, B, Hq, Hkv, part):
    c = make_random_case("fused", Hq, Hkv, D, B, LENS, DT[dt], seed=D + B + Hq, device=DEV,
                         with_append=True)
    fused_vs_oracle(c, part, f"{dt} D{D} B{B} G{Hq // Hkv} p{part}")


def test_fused_append_auto_partition():
    c = make_random_case("fused_auto", 32, 8, 128, 16, [4096, 50, 1], torch.bfloat16, seed=9,
                         device=DEV, with_append=True)
    fused_vs_oracle(c, pkv.PARTITION_AUTO, "fused, auto partition")


def test_fused_append_opt13b_workload():
    c = make_case("opt13b_mha_b64", device=DEV)
    fused_vs_oracle(c, c.partition_size, "opt13b fused")


def test_fused_append_shared_prefix_pipeline():
    sp = make_shared_prefix_case(device=DEV, decode_steps=20)
    kc, vc = sp.k_pool.cpu(), sp.v_pool.cpu()
    pkv.kv_block_copy(sp.k_pool, sp.v_pool, sp.cow_pairs)
    oracle.block_copy(kc, vc, sp.cow_pairs.cpu())
    for k, st in enumerate(sp.steps):
        q, kn, vn = sp.step_tokens(k)
        out = torch.empty_like(q)
        pkv.paged_attn_decode_append(out, q, kn, vn, sp.k_pool, sp.v_pool, st["block_tables"],
                                     st["context_lens"], sp.scale,
                                     int(st["context_lens"].max()), partition_size=512)
        oracle.cache_append(kc, vc, kn.cpu(), vn.cpu(), st["slot_mapping"].cpu())
        if k in (0, 7, 19):
            ref = oracle.paged_decode(q.cpu(), kc, vc, st["block_tables"].cpu(),
                                      st["context_lens"].cpu(), sp.scale)
            assert_close_to_oracle(out, ref, torch.float16, f"shared prefix fused step {k}")
    torch.cuda.synchronize()
    assert torch.equal(sp.k_pool.cpu().view(torch.int16), kc.view(torch.int16))
    assert torch.equal(sp.v_pool.cpu().view(torch.int16), vc.view(torch.int16))


def test_fused_append_rejects_fp32():
    c = make_random_case("f32", 2, 2, 64, 16, [5], torch.float32, seed=1, device=DEV,
                         with_append=True)
    out = torch.empty_like(c.q)
    with pytest.raises(pkv.PkvError) as e:
        pkv.paged_attn_decode_append(out, c.q, c.k_new, c.v_new, c.k_pool, c.v_pool,
                                     c.block_tables, c.context_lens, c.scale, 5)
    assert e.value.status == pkv.PKV_EUNSUPPORTED


@pytest.mark.parametrize("fused", [False, True])
@pytest.mark.parametrize("part", [0, 512])
def test_output_into_pinned_host_memory(fused, part):
    """`out` may be page-locked host memory: the kernels write it over the bus,
    bit for bit what they write into device memory (merged partitions included)."""
    c = make_random_case("pinned_out", 16, 4, 128, 16, LENS, torch.bfloat16, seed=7, device=DEV,
                         with_append=True)
    if not fused:
        pkv.kv_cache_append(c.k_pool, c.v_pool, c.k_new, c.v_new, c.slot_mapping)
    dev_out = torch.empty_like(c.q)
    host_out = torch.full(tuple(c.q.shape), float("nan"), dtype=c.q.dtype).pin_memory()
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    for o in (dev_out, host_out):
        if fused:  # appending the same token twice leaves the pool unchanged
            pkv.paged_attn_decode_append(o, c.q, c.k_new, c.v_new, c.k_pool, c.v_pool,
                                         c.block_tables, c.context_lens, c.scale,
                                         c.max_context_len, partition_size=part, err=err)
        else:
            pkv.paged_attn_decode(o, c.q, c.k_pool, c.v_pool, c.block_tables, c.context_lens,
                                  c.scale, c.max_context_len, partition_size=part, err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert torch.equal(dev_out.cpu().view(torch.int16), host_out.view(torch.int16))


@pytest.mark.parametrize("part", [0, 64])
def test_lengths_advanced_on_device_just_before_each_call(part):
    """A serving loop advances the context lengths with a device kernel on the
    same stream right before each fused call. Every call must attend over the
    new lengths and append at the new last slot."""
    Hq, Hkv, D, B, S, steps = 8, 2, 128, 16, 24, 6
    dt = torch.bfloat16
    g = torch.Generator().manual_seed(11)
    lens0 = torch.randint(1, 200, (S,), generator=g, dtype=torch.int32)
    maxlen = int(lens0.max()) + steps
    nb = -(-maxlen // B)
    tables = torch.randperm(S * nb, generator=g).to(torch.int32).view(S, nb)
    kc = torch.randn(S * nb, Hkv, B, D, generator=g).to(dt)
    vc = torch.randn(S * nb, Hkv, B, D, generator=g).to(dt)
    kd, vd, bt = kc.to(DEV), vc.to(DEV), tables.to(DEV)
    lens = (lens0 - 1).to(DEV)  # the loop adds one before each call
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    for step in range(steps):
        q = torch.randn(S, Hq, D, generator=g).to(dt)
        kn = torch.randn(S, Hkv, D, generator=g).to(dt)
        vn = torch.randn(S, Hkv, D, generator=g).to(dt)
        qd, knd, vnd = q.to(DEV), kn.to(DEV), vn.to(DEV)
        out = torch.empty_like(qd)
        lens.add_(1)  # the kernel just before the call writes the lengths
        pkv.paged_attn_decode_append(out, qd, knd, vnd, kd, vd, bt, lens, D ** -0.5, maxlen,
                                     partition_size=part, err=err)
        L = (lens0 + step).to(torch.int64)
        slots = tables[torch.arange(S), (L - 1) // B].to(torch.int64) * B + (L - 1) % B
        oracle.cache_append(kc, vc, kn, vn, slots)
        ref = oracle.paged_decode(q, kc, vc, tables, L.to(torch.int32), D ** -0.5)
        torch.cuda.synchronize()
        assert int(err.item()) == 0, f"step {step}"
        assert_close_to_oracle(out, ref, dt, f"device-advanced lengths, step {step}")
    assert torch.equal(kd.cpu().view(torch.int16), kc.view(torch.int16))
    assert torch.equal(vd.cpu().view(torch.int16), vc.view(torch.int16))


# ---------------------------------------------------------------------------
# the timed workloads at full size, every output, through the benchmarked call
# ---------------------------------------------------------------------------

def test_full_batch256_gqa_step_as_benchmarked():
    """The batch-256 GQA step exactly as the benchmark times it: one
    paged_attn_decode_append call with 2048-token partitions. All 256
    sequences' outputs (every query head, every element) are compared with the
    oracle's decode over the appended cache, and both pools with the oracle's
    append, bit for bit (page "PagedAttention", newikis, section "Mathematical
    formulation"; page "PagedAttention Analysis", section 3: the block-wise
    walk equals ordinary attention)."""
    c = make_case("llama8b_gqa_b256", device=DEV, with_append=True)
    assert c.num_seqs == 256 and c.partition_size == 2048
    fused_vs_oracle(c, c.partition_size, "batch-256 GQA, full batch, fused")


def test_full_long_split_step_as_benchmarked():
    """The long-context workload (8 sequences of 32768-131072 tokens, block 32)
    at its 512-token partitions, through the fused call the benchmark times:
    every output of all 8 sequences against the oracle, pools bit-exact. Each
    context spans 64-256 partitions, so every one goes through the two-level
    log-sum-exp merge."""
    c = make_case("long_split_b8", device=DEV, with_append=True)
    assert c.num_seqs == 8 and c.partition_size == 512
    assert int(c.context_lens.min()) > 16 * 512  # more than one merge chunk each
    fused_vs_oracle(c, c.partition_size, "long split, all 8 sequences, fused")
