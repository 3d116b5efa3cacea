"""Shared helpers for the parity tests: run the CUDA path, run the oracle,
compare with the acceptance tolerances."""

from __future__ import annotations

import numpy as np
import torch

import oracle
import paged_kv_cache_387_b200 as pkv

# Acceptance tolerances: |err| <= ABS + REL*|ref| for 16-bit inputs with fp32
# accumulation, and |err| <= 1e-5 for fp32 inputs.
TOL_16 = (2e-3, 1e-2)
TOL_32 = (1e-5, 0.0)


def tolerance(dtype):
    return TOL_32 if dtype == torch.float32 else TOL_16


def assert_close_to_oracle(got: torch.Tensor, ref: np.ndarray, dtype, what=""):
    g = got.detach().to("cpu", torch.float64).numpy()
    assert g.shape == ref.shape, (g.shape, ref.shape)
    assert not np.isnan(g).any(), f"{what}: NaN in kernel output"
    a, r = tolerance(dtype)
    err = np.abs(g - ref)
    bound = a + r * np.abs(ref)
    bad = err > bound
    if bad.any():
        idx = np.argwhere(bad)[0]
        raise AssertionError(f"{what}: {int(bad.sum())} of {bad.size} outside tolerance; "
                             f"first at {tuple(idx)}: got {g[tuple(idx)]}, ref {ref[tuple(idx)]}, "
                             f"max err {err.max():.3e}")
    return float(err.max())


def gpu_decode(case, partition_size=None, err=None, max_context_len=None):
    out = torch.empty_like(case.q)
    ps = case.partition_size if partition_size is None else partition_size
    mcl = case.max_context_len if max_context_len is None else max_context_len
    pkv.paged_attn_decode(out, case.q, case.k_pool, case.v_pool, case.block_tables,
                          case.context_lens, case.scale, mcl, partition_size=ps, err=err)
    return out


def oracle_decode(case, seqs=None):
    """Oracle output for all sequences, or for the listed subset."""
    q, bt, cl = case.q.cpu(), case.block_tables.cpu(), case.context_lens.cpu()
    kp = case.k_pool if case.k_pool.device.type == "cpu" else case.k_pool.cpu()
    vp = case.v_pool if case.v_pool.device.type == "cpu" else case.v_pool.cpu()
    if seqs is not None:
        idx = torch.as_tensor(seqs, dtype=torch.long)
        q, bt, cl = q[idx].contiguous(), bt[idx].contiguous(), cl[idx].contiguous()
    return oracle.paged_decode(q, kp, vp, bt, cl, case.scale)


def new_err(device):
    return torch.zeros(1, dtype=torch.int32, device=device)
