"""Byte counts for the bandwidth figures (measurement arithmetic only)."""

from __future__ import annotations

from typing import Iterable


def kv_bytes_per_token(num_layers: int, num_kv_heads: int, head_dim: int,
                       elem_bytes: int) -> int:
    """K and V bytes one token occupies across all layers: 2*L*Hkv*D*sz.

    For a 13B OPT model (40 layers, 40 heads of 128, fp16) this is 819,200 B,
    which is 800 KiB. Page "PagedAttention Analysis", section 1, gives about
    800KB per token for that model.
    """
    return 2 * num_layers * num_kv_heads * head_dim * elem_bytes


def decode_algorithmic_bytes(context_lens: Iterable[int], num_heads: int,
                             num_kv_heads: int, head_dim: int, block_size: int,
                             elem_bytes: int) -> int:
    """Minimum bytes one decode step over one layer must move.

    Per sequence of length L:
      K and V of every valid token, once per KV head: 2*L*Hkv*D*sz
      q in and o out:                                2*Hq*D*sz
      its block-table entries and context length:     4*ceil(L/B) + 4
    Reserved-but-empty slots and split-context workspace are excluded.
    """
    total = 0
    for L in context_lens:
        L = int(L)
        nb = -(-L // block_size)
        total += 2 * L * num_kv_heads * head_dim * elem_bytes
        total += 2 * num_heads * head_dim * elem_bytes
        total += 4 * nb + 4
    return total


def unique_kv_bytes(block_tables, context_lens, block_size: int, num_kv_heads: int,
                    head_dim: int, elem_bytes: int) -> int:
    """K and V bytes of the distinct physical blocks a decode step reads.

    Sequences that share a block (forked samples, beams, cached prefixes) read
    the same memory; counted once, with the most slots any of them reads from
    it. This is the traffic a reader that fetches each shared block once must
    move, the bound for the sharing workloads; the per-sequence sum of
    decode_algorithmic_bytes counts a shared block once per reader.
    """
    best = {}
    for row, L in zip(block_tables, context_lens):
        L = int(L)
        for j in range(-(-L // block_size)):
            b = int(row[j])
            n = min(block_size, L - j * block_size)
            if n > best.get(b, 0):
                best[b] = n
    return sum(best.values()) * 2 * num_kv_heads * head_dim * elem_bytes
