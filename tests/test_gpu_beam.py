"""Beam search through the CUDA path against the oracle, step by step: the
beams share the prompt and intermediate blocks and the sharing changes every
step (page "PagedAttention Analysis", section 4). Each step runs the
copy-on-write block copies (kv_block_copy), then the fused append + decode;
the oracle runs its block copy, cache append and decode. The pools must agree
bit for bit and the outputs within the tolerance."""

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_387_b200 as pkv
from pkv_inputs import BeamSearch, BlockAllocator
from tests.helpers import assert_close_to_oracle, new_err

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("dt,B,Hq,Hkv,D", [(torch.bfloat16, 16, 8, 2, 128),
                                          (torch.float16, 8, 4, 4, 64)])
def test_beam_search_steps_match_oracle(dt, B, Hq, Hkv, D):
    R, W, prompt, steps = 2, 4, 40, 25
    P = R * W * (-(-(prompt + steps) // B) + 1)
    rng = np.random.default_rng(17)
    g = torch.Generator().manual_seed(17)
    alloc = BlockAllocator(P, B, free_order=rng.permutation(P).tolist())
    kd = torch.full((P, Hkv, B, D), float("nan"), dtype=dt, device=DEV)
    vd = torch.full_like(kd, float("nan"))
    kc, vc = kd.cpu(), vd.cpu()  # the oracle's pools
    err = new_err(DEV)
    searches = []
    for _ in range(R):
        bs = BeamSearch(alloc, prompt, W)
        t = np.arange(prompt)
        slots = torch.as_tensor(np.asarray(bs.beams[0].table)[t // B] * B + t % B)
        kt = torch.randn(prompt, Hkv, D, generator=g).to(dt)
        vt = torch.randn(prompt, Hkv, D, generator=g).to(dt)
        pkv.kv_cache_append(kd, vd, kt.to(DEV), vt.to(DEV), slots.to(DEV), err=err)
        oracle.cache_append(kc, vc, kt, vt, slots)
        searches.append(bs)
    for step in range(steps):
        slots, copies = [], []
        for bs in searches:
            s, c = bs.step(rng.integers(0, W, size=W))
            slots += s
            copies += c
        if copies:
            pairs = torch.tensor([[c.src, c.dst] for c in copies], dtype=torch.int32)
            pkv.kv_block_copy(kd, vd, pairs.to(DEV), err=err)
            oracle.block_copy(kc, vc, pairs.numpy())
        beams = [b for bs in searches for b in bs.beams]
        S = len(beams)
        bt = torch.full((S, max(len(b.table) for b in beams)), -1, dtype=torch.int32)
        for i, b in enumerate(beams):
            bt[i, :len(b.table)] = torch.tensor(b.table, dtype=torch.int32)
        lens = torch.tensor([b.num_tokens for b in beams], dtype=torch.int32)
        q = torch.randn(S, Hq, D, generator=g).to(dt)
        kn = torch.randn(S, Hkv, D, generator=g).to(dt)
        vn = torch.randn(S, Hkv, D, generator=g).to(dt)
        out = torch.empty(S, Hq, D, dtype=dt, device=DEV)
        pkv.paged_attn_decode_append(out, q.to(DEV), kn.to(DEV), vn.to(DEV), kd, vd, bt.to(DEV),
                                     lens.to(DEV), 1.0 / D ** 0.5, int(lens.max()),
                                     partition_size=16 if step % 2 else 0, err=err)
        oracle.cache_append(kc, vc, kn, vn, torch.tensor(slots, dtype=torch.int64))
        ref = oracle.paged_decode(q, kc, vc, bt, lens, 1.0 / D ** 0.5)
        torch.cuda.synchronize()
        assert int(err.item()) == 0, f"step {step}"
        assert torch.equal(kd.cpu().view(torch.int16), kc.view(torch.int16)), f"step {step}"
        assert torch.equal(vd.cpu().view(torch.int16), vc.view(torch.int16)), f"step {step}"
        assert_close_to_oracle(out, ref, dt, f"beam step {step}")
    for bs in searches:
        bs.release()
    assert alloc.num_free == P
