"""Pins for the CPU oracle: each check ties it to something other than itself.

* A library routine. Paged attention must equal ordinary attention over
  contiguous K/V; page "PagedAttention Analysis", section 3, says the block-wise
  form is mathematically identical. The contiguous side here is PyTorch's
  ``scaled_dot_product_attention`` in float64 on arrays that were never paged.
* Invariants. The result is unchanged under any physical block placement:
  page "PagedAttention" (newikis), section "Mathematical formulation", says
  blocks may sit anywhere in physical memory. Poisoned unused slots have no
  effect, and GQA equals MHA with repeated KV heads.
* Closed forms. One token gives o = v. Equal keys, or a zero scale, give
  o = mean(V).
* Agreement of the oracle's three forms: the definition (two-pass), the
  pages' block-by-block online-softmax walk, and split partitions combined by
  log-sum-exp.
* Exhaustive checks of the bit decoders against numpy's and torch's
  conversions.
"""

import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from hypothesis import given, settings
from hypothesis import strategies as st

import oracle

DT = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}


def dense_tokens(lens, Hkv, D, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    ks = [torch.randn(L, Hkv, D, generator=g).to(dtype) for L in lens]
    vs = [torch.randn(L, Hkv, D, generator=g).to(dtype) for L in lens]
    return ks, vs


def page_tokens(ks, vs, B, num_blocks, perm, fill=float("nan")):
    """Write each sequence's dense tokens into a pool block by block, taking
    physical blocks in the order given by ``perm`` (plain loops, tiny sizes)."""
    Hkv, D = ks[0].shape[1], ks[0].shape[2]
    dtype = ks[0].dtype
    k_pool = torch.full((num_blocks, Hkv, B, D), fill, dtype=dtype)
    v_pool = torch.full((num_blocks, Hkv, B, D), fill, dtype=dtype)
    tables = []
    nxt = 0
    for k, v in zip(ks, vs):
        L = k.shape[0]
        row = []
        for j in range(-(-L // B)):
            phys = int(perm[nxt])
            nxt += 1
            row.append(phys)
            for t in range(j * B, min(L, (j + 1) * B)):
                k_pool[phys, :, t - j * B, :] = k[t]
                v_pool[phys, :, t - j * B, :] = v[t]
        tables.append(row)
    mb = max(1, max(len(r) for r in tables))
    bt = torch.full((len(ks), mb), -1, dtype=torch.int32)
    for s, r in enumerate(tables):
        bt[s, :len(r)] = torch.tensor(r, dtype=torch.int32)
    lens = torch.tensor([k.shape[0] for k in ks], dtype=torch.int32)
    return k_pool, v_pool, bt, lens


def sdpa_reference(q, ks, vs, scale):
    """Contiguous attention per sequence through torch SDPA in float64."""
    S, Hq, D = q.shape
    out = np.zeros((S, Hq, D))
    for s in range(S):
        k = ks[s].double().permute(1, 0, 2)  # [Hkv][L][D]
        v = vs[s].double().permute(1, 0, 2)
        G = Hq // k.shape[0]
        k = k.repeat_interleave(G, dim=0)
        v = v.repeat_interleave(G, dim=0)
        qs = q[s].double().unsqueeze(1)       # [Hq][1][D]
        o = F.scaled_dot_product_attention(qs, k, v, scale=scale)
        out[s] = o.squeeze(1).numpy()
    return out


CASES = [
    # (lens, Hq, Hkv, D, B, dtype)
    ([1, 15, 16, 37], 2, 2, 64, 16, "f32"),
    ([5, 33, 64, 100], 8, 2, 64, 16, "bf16"),
    ([17, 3, 48], 4, 1, 128, 32, "f16"),
    ([9, 1, 40], 6, 3, 32, 8, "f32"),
]


@pytest.mark.parametrize("lens,Hq,Hkv,D,B,dt", CASES)
def test_paged_equals_contiguous_library_attention(lens, Hq, Hkv, D, B, dt):
    dtype = DT[dt]
    ks, vs = dense_tokens(lens, Hkv, D, dtype, seed=7)
    q = torch.randn(len(lens), Hq, D, generator=torch.Generator().manual_seed(8)).to(dtype)
    nb = sum(-(-L // B) for L in lens) + 5
    perm = np.random.default_rng(3).permutation(nb)
    k_pool, v_pool, bt, cl = page_tokens(ks, vs, B, nb, perm)
    scale = 1.0 / math.sqrt(D)
    got = oracle.paged_decode(q, k_pool, v_pool, bt, cl, scale)
    ref = sdpa_reference(q, ks, vs, scale)
    assert np.abs(got - ref).max() < 1e-12


def test_placement_permutation_invariance():
    lens, Hq, Hkv, D, B = [3, 29, 50, 16], 4, 2, 64, 16
    ks, vs = dense_tokens(lens, Hkv, D, torch.bfloat16, seed=11)
    q = torch.randn(len(lens), Hq, D, generator=torch.Generator().manual_seed(12)).bfloat16()
    nb = 40
    outs = []
    for seed in (0, 1, 2):
        perm = np.random.default_rng(seed).permutation(nb)
        k_pool, v_pool, bt, cl = page_tokens(ks, vs, B, nb, perm)
        outs.append(oracle.paged_decode(q, k_pool, v_pool, bt, cl, 0.125))
    # same arithmetic in the same order: identical bits
    assert np.array_equal(outs[0], outs[1]) and np.array_equal(outs[0], outs[2])


def test_single_token_returns_its_value():
    ks, vs = dense_tokens([1, 1], 2, 64, torch.float16, seed=5)
    q = torch.randn(2, 4, 64).half() * 10
    k_pool, v_pool, bt, cl = page_tokens(ks, vs, 16, 4, [3, 1, 0, 2])
    got = oracle.paged_decode(q, k_pool, v_pool, bt, cl, 1 / 8)
    for s in range(2):
        for h in range(4):
            assert np.array_equal(got[s, h], vs[s][0, h // 2].double().numpy())


def test_equal_keys_or_zero_scale_give_mean_of_values():
    lens = [7, 33]
    ks, vs = dense_tokens(lens, 1, 64, torch.float32, seed=2)
    ks = [torch.ones_like(k) * 0.5 for k in ks]
    q = torch.randn(2, 3, 64)
    k_pool, v_pool, bt, cl = page_tokens(ks, vs, 16, 8, np.arange(8)[::-1].copy())
    got = oracle.paged_decode(q, k_pool, v_pool, bt, cl, 1 / 8)
    for s, L in enumerate(lens):
        mean = vs[s][:, 0].double().mean(0).numpy()
        assert np.abs(got[s] - mean[None]).max() < 1e-13
    # random keys, scale 0: every score is 0
    ks, _ = dense_tokens(lens, 1, 64, torch.float32, seed=9)
    k_pool, v_pool, bt, cl = page_tokens(ks, vs, 16, 8, np.arange(8))
    got = oracle.paged_decode(q, k_pool, v_pool, bt, cl, 0.0)
    for s, L in enumerate(lens):
        assert np.abs(got[s] - vs[s][:, 0].double().mean(0).numpy()[None]).max() < 1e-13


@pytest.mark.parametrize("dt", ["f32", "f16", "bf16"])
def test_blockwise_walk_matches_definition(dt):
    from pkv_inputs import make_random_case
    c = make_random_case("pin", 8, 2, 64, 16, [1, 15, 16, 17, 37, 130, 260], DT[dt], seed=4,
                         pool_blocks=60)
    a = oracle.paged_decode(c.q, c.k_pool, c.v_pool, c.block_tables, c.context_lens, c.scale)
    b = oracle.paged_decode_blockwise(c.q, c.k_pool, c.v_pool, c.block_tables, c.context_lens,
                                      c.scale)
    assert not np.isnan(a).any()
    assert np.abs(a - b).max() < 1e-12


@pytest.mark.parametrize("part", [16, 32, 48, 512])
def test_partition_lse_merge_matches_unsplit(part):
    from pkv_inputs import make_random_case
    c = make_random_case("pin", 4, 4, 64, 16, [1, 16, 47, 200, 513], torch.bfloat16, seed=6)
    a, lse = oracle.paged_decode(c.q, c.k_pool, c.v_pool, c.block_tables, c.context_lens,
                                 c.scale, return_lse=True)
    b, po, pl = oracle.paged_decode_partitioned(c.q, c.k_pool, c.v_pool, c.block_tables,
                                                c.context_lens, c.scale, part)
    assert np.abs(a - b).max() < 1e-12
    # the partitions' lse combine to the whole context's lse
    comb = np.log(np.exp(pl).sum(-1))
    assert np.abs(comb - lse).max() < 1e-12


def test_poisoned_slots_do_not_reach_the_output():
    from pkv_inputs import make_random_case
    kw = dict(name="pin", num_heads=4, num_kv_heads=2, head_dim=64, block_size=16,
              context_lens=[1, 15, 33], dtype=torch.float16, seed=21, pool_blocks=12)
    a = make_random_case(poison=True, **kw)
    b = make_random_case(poison=False, **kw)
    assert torch.isnan(a.k_pool).any()
    oa = oracle.paged_decode(a.q, a.k_pool, a.v_pool, a.block_tables, a.context_lens, a.scale)
    ob = oracle.paged_decode(b.q, b.k_pool, b.v_pool, b.block_tables, b.context_lens, b.scale)
    assert not np.isnan(oa).any()
    assert np.array_equal(oa, ob)


def test_gqa_equals_mha_with_repeated_kv_heads():
    from pkv_inputs import make_random_case
    c = make_random_case("pin", 8, 2, 64, 16, [5, 40, 77], torch.bfloat16, seed=31)
    G = 4
    k_rep = c.k_pool.repeat_interleave(G, dim=1).contiguous()
    v_rep = c.v_pool.repeat_interleave(G, dim=1).contiguous()
    a = oracle.paged_decode(c.q, c.k_pool, c.v_pool, c.block_tables, c.context_lens, c.scale)
    b = oracle.paged_decode(c.q, k_rep, v_rep, c.block_tables, c.context_lens, c.scale)
    assert np.array_equal(a, b)


def test_bad_block_id_is_reported():
    from pkv_inputs import make_random_case
    c = make_random_case("pin", 2, 2, 64, 16, [20], torch.float32, seed=1)
    bt = c.block_tables.clone()
    bt[0, 1] = c.num_blocks  # out of range
    with pytest.raises(RuntimeError):
        oracle.paged_decode(c.q, c.k_pool, c.v_pool, bt, c.context_lens, c.scale)


def test_half_decoder_exhaustive():
    bits = np.arange(1 << 16, dtype=np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([oracle.half_to_double(int(b)) for b in bits])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


def test_bf16_decoder_exhaustive():
    bits = torch.arange(1 << 16, dtype=torch.int32).to(torch.int16)
    ref = bits.view(torch.bfloat16).double().numpy()
    got = np.array([oracle.bf16_to_double(int(b) & 0xFFFF) for b in range(1 << 16)])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


def test_append_matches_numpy_scatter():
    rng = np.random.default_rng(5)
    P, Hkv, B, D, T = 10, 3, 16, 64, 12
    k_pool = torch.from_numpy(rng.standard_normal((P, Hkv, B, D)).astype(np.float32)).half()
    v_pool = torch.from_numpy(rng.standard_normal((P, Hkv, B, D)).astype(np.float32)).half()
    k_new = torch.from_numpy(rng.standard_normal((T, Hkv, D)).astype(np.float32)).half()
    v_new = torch.from_numpy(rng.standard_normal((T, Hkv, D)).astype(np.float32)).half()
    slots = rng.choice(P * B, size=T, replace=False).astype(np.int64)
    slots[3] = -1  # skipped
    ek, ev = k_pool.numpy().copy(), v_pool.numpy().copy()
    m = slots >= 0
    ek[slots[m] // B, :, slots[m] % B, :] = k_new.numpy()[m]
    ev[slots[m] // B, :, slots[m] % B, :] = v_new.numpy()[m]
    oracle.cache_append(k_pool, v_pool, k_new, v_new, torch.from_numpy(slots))
    assert np.array_equal(k_pool.numpy().view(np.uint16), ek.view(np.uint16))
    assert np.array_equal(v_pool.numpy().view(np.uint16), ev.view(np.uint16))


def test_block_copy_matches_numpy_slices():
    rng = np.random.default_rng(8)
    P, Hkv, B, D = 12, 2, 16, 64
    k_pool = torch.from_numpy(rng.standard_normal((P, Hkv, B, D)).astype(np.float32)).bfloat16()
    v_pool = torch.from_numpy(rng.standard_normal((P, Hkv, B, D)).astype(np.float32)).bfloat16()
    pairs = np.array([[1, 7], [4, 9], [1, 11]], dtype=np.int32)
    ek = k_pool.view(torch.int16).numpy().copy()
    ev = v_pool.view(torch.int16).numpy().copy()
    for s, d in pairs:
        ek[d] = ek[s]
        ev[d] = ev[s]
    oracle.block_copy(k_pool, v_pool, torch.from_numpy(pairs))
    assert np.array_equal(k_pool.view(torch.int16).numpy(), ek)
    assert np.array_equal(v_pool.view(torch.int16).numpy(), ev)


def test_append_out_of_range_slot_is_skipped_and_reported():
    """A slot at or past num_blocks * B names no pool slot: the oracle skips that
    token, still writes every other token (the numpy scatter of the valid ones)
    and reports the error."""
    rng = np.random.default_rng(6)
    P, Hkv, B, D, T = 6, 2, 8, 16, 5
    k_pool = torch.from_numpy(rng.standard_normal((P, Hkv, B, D)).astype(np.float32)).bfloat16()
    v_pool = torch.from_numpy(rng.standard_normal((P, Hkv, B, D)).astype(np.float32)).bfloat16()
    k_new = torch.from_numpy(rng.standard_normal((T, Hkv, D)).astype(np.float32)).bfloat16()
    v_new = torch.from_numpy(rng.standard_normal((T, Hkv, D)).astype(np.float32)).bfloat16()
    slots = np.array([3, P * B, 17, P * B + 40, P * B - 1], dtype=np.int64)
    ek = k_pool.view(torch.int16).numpy().copy()
    ev = v_pool.view(torch.int16).numpy().copy()
    for i, sl in enumerate(slots):
        if sl < P * B:
            ek[sl // B, :, sl % B, :] = k_new.view(torch.int16).numpy()[i]
            ev[sl // B, :, sl % B, :] = v_new.view(torch.int16).numpy()[i]
    with pytest.raises(RuntimeError, match="out of range"):
        oracle.cache_append(k_pool, v_pool, k_new, v_new, torch.from_numpy(slots))
    assert np.array_equal(k_pool.view(torch.int16).numpy(), ek)
    assert np.array_equal(v_pool.view(torch.int16).numpy(), ev)


@pytest.mark.parametrize("bad", [[12, 3], [-1, 3], [2, 12], [2, -5]])
def test_block_copy_out_of_range_pair_is_skipped_and_reported(bad):
    """A pair whose source or destination lies outside [0, num_blocks) is
    skipped and reported; the in-range pairs around it are still copied."""
    rng = np.random.default_rng(9)
    P, Hkv, B, D = 12, 2, 16, 32
    k_pool = torch.from_numpy(rng.standard_normal((P, Hkv, B, D)).astype(np.float32)).half()
    v_pool = torch.from_numpy(rng.standard_normal((P, Hkv, B, D)).astype(np.float32)).half()
    pairs = np.array([[1, 7], bad, [4, 9]], dtype=np.int32)
    ek = k_pool.view(torch.int16).numpy().copy()
    ev = v_pool.view(torch.int16).numpy().copy()
    for s_, d_ in ([1, 7], [4, 9]):
        ek[d_] = ek[s_]
        ev[d_] = ev[s_]
    with pytest.raises(RuntimeError, match="out of range"):
        oracle.block_copy(k_pool, v_pool, torch.from_numpy(pairs))
    assert np.array_equal(k_pool.view(torch.int16).numpy(), ek)
    assert np.array_equal(v_pool.view(torch.int16).numpy(), ev)


def test_block_swap_is_numpy_block_assignment():
    """oracle.block_swap copies whole blocks between two pools: the same as
    torch's indexed assignment dst[d] = src[s] per pair, bit for bit."""
    import torch
    rng = np.random.default_rng(11)
    for dt in (torch.float16, torch.bfloat16, torch.float32):
        src_k = torch.from_numpy(rng.standard_normal((9, 2, 16, 64)).astype(np.float32)).to(dt)
        src_v = torch.from_numpy(rng.standard_normal((9, 2, 16, 64)).astype(np.float32)).to(dt)
        dst_k = torch.full((6, 2, 16, 64), float("nan"), dtype=dt)
        dst_v = torch.full_like(dst_k, float("nan"))
        pairs = np.array([[7, 0], [2, 5], [7, 3], [0, 1]], dtype=np.int32)
        ek, ev = dst_k.clone(), dst_v.clone()
        for s_, d_ in pairs:
            ek[d_] = src_k[s_]
            ev[d_] = src_v[s_]
        oracle.block_swap(dst_k, dst_v, src_k, src_v, pairs)
        bits = torch.int32 if dt == torch.float32 else torch.int16
        assert torch.equal(dst_k.view(bits), ek.view(bits))
        assert torch.equal(dst_v.view(bits), ev.view(bits))
        with pytest.raises(RuntimeError):
            oracle.block_swap(dst_k, dst_v, src_k, src_v, np.array([[9, 0]], dtype=np.int32))


@settings(max_examples=60, deadline=None)
@given(lens=st.lists(st.integers(1, 70), min_size=1, max_size=4),
       B=st.sampled_from([1, 3, 8, 16]), Hkv=st.integers(1, 2), G=st.integers(1, 3),
       D=st.sampled_from([8, 16, 64]), dt=st.sampled_from(["f32", "f16", "bf16"]),
       scale=st.floats(0.0, 1.0), seed=st.integers(0, 2 ** 16), part=st.sampled_from([1, 5, 32]))
def test_random_shapes_equal_contiguous_library_attention(lens, B, Hkv, G, D, dt, scale, seed,
                                                           part):
    """The library-routine pin over random shapes, block sizes, group sizes,
    dtypes, scales and placements; the partitioned form (partitions of `part`
    blocks) agrees too."""
    dtype = DT[dt]
    ks, vs = dense_tokens(lens, Hkv, D, dtype, seed=seed)
    q = torch.randn(len(lens), Hkv * G, D,
                    generator=torch.Generator().manual_seed(seed + 1)).to(dtype)
    nb = sum(-(-L // B) for L in lens) + 3
    perm = np.random.default_rng(seed).permutation(nb)
    k_pool, v_pool, bt, cl = page_tokens(ks, vs, B, nb, perm)
    got = oracle.paged_decode(q, k_pool, v_pool, bt, cl, scale)
    ref = sdpa_reference(q, ks, vs, scale)
    assert np.abs(got - ref).max() < 1e-12
    split, _, _ = oracle.paged_decode_partitioned(q, k_pool, v_pool, bt, cl, scale, part * B)
    assert np.abs(split - got).max() < 1e-12
