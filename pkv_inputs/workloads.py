"""Seeded decode workloads: q, paged K/V pools, block tables, lengths, slots.

Pool layout (shared by every producer and consumer of the pools):

    k_pool[phys_block][kv_head][slot][d]   (same for v_pool)

This is row-major with ``d`` contiguous. Token ``t`` of a sequence whose
block table is ``bt`` lives at ``phys_block = bt[t // B]`` and
``slot = t % B``. The slot mapping used by cache-append addresses
``phys_block * B + slot``.

Shapes follow the decode workloads the pages discuss: OPT-13B-shaped heads
(page "PagedAttention Analysis", section 1) and LLaMA-class GQA heads, 16-token
blocks (the default block size in that page's section 6), ragged lengths, and
prompts shared by parallel samples (same page, section 4). All values are
synthetic. The pages measure on ShareGPT/Alpaca traces with real model weights,
which are not used here. Seeded N(0,1) values and seeded length distributions
stand in for them.

Poisoning. Every pool slot that no valid token occupies is filled with NaN:
the unassigned blocks, the tail of each last block, and the slot a pending
append will write. Any consumer that reads a masked slot into its result
therefore shows it as a NaN.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field, replace
from typing import Dict, List, Optional, Sequence

import numpy as np
import torch

from .block_manager import BeamSearch, BlockAllocator, PrefixCache

POOL_LAYOUT = "[num_blocks][num_kv_heads][block_size][head_dim], head_dim contiguous"

DTYPES = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}
DTYPE_NAMES = {v: k for k, v in DTYPES.items()}

# Tokens per split-context partition. 2048 is the library default. The
# long-context workload is specified with 512-token partitions and keeps them.
DEFAULT_PARTITION = 2048
LONG_CONTEXT_PARTITION = 512


def nan_fill_value(dtype: torch.dtype) -> float:
    return float("nan")


@dataclass
class DecodeCase:
    """One decode step's inputs (plus the optional append that precedes it)."""

    name: str
    q: torch.Tensor               # [S][Hq][D]
    k_pool: torch.Tensor          # [P][Hkv][B][D]
    v_pool: torch.Tensor          # [P][Hkv][B][D]
    block_tables: torch.Tensor    # int32 [S][max_blocks], padding -1
    context_lens: torch.Tensor    # int32 [S]
    num_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    scale: float
    partition_size: int = DEFAULT_PARTITION
    k_new: Optional[torch.Tensor] = None        # [T][Hkv][D]
    v_new: Optional[torch.Tensor] = None        # [T][Hkv][D]
    slot_mapping: Optional[torch.Tensor] = None  # int64 [T]
    meta: Dict = field(default_factory=dict)

    @property
    def num_seqs(self) -> int:
        return int(self.q.shape[0])

    @property
    def num_blocks(self) -> int:
        return int(self.k_pool.shape[0])

    @property
    def max_blocks_per_seq(self) -> int:
        return int(self.block_tables.shape[1])

    @property
    def max_context_len(self) -> int:
        return int(self.context_lens.max().item()) if self.num_seqs else 0

    @property
    def dtype(self) -> torch.dtype:
        return self.q.dtype

    def to(self, device) -> "DecodeCase":
        def mv(t):
            return None if t is None else t.to(device)
        return replace(self, q=mv(self.q), k_pool=mv(self.k_pool), v_pool=mv(self.v_pool),
                       block_tables=mv(self.block_tables), context_lens=mv(self.context_lens),
                       k_new=mv(self.k_new), v_new=mv(self.v_new),
                       slot_mapping=mv(self.slot_mapping))


def _generator(seed: int, device) -> torch.Generator:
    dev = torch.device(device)
    g = torch.Generator(device=dev)
    g.manual_seed(int(seed))
    return g


def _randn(shape, gen: torch.Generator, dtype: torch.dtype, device,
           chunk_elems: int = 1 << 24) -> torch.Tensor:
    """N(0,1) draws rounded to ``dtype``; generated in chunks to bound fp32 temporaries."""
    out = torch.empty(shape, dtype=dtype, device=device)
    flat = out.view(-1)
    n = flat.numel()
    for i in range(0, n, chunk_elems):
        j = min(n, i + chunk_elems)
        flat[i:j] = torch.randn(j - i, generator=gen, device=device, dtype=torch.float32).to(dtype)
    return out


def _place_blocks(context_lens: np.ndarray, block_size: int, pool_blocks: int,
                  rng: np.random.Generator, placement: str) -> np.ndarray:
    """Block tables: sequence s's logical blocks take consecutive entries of a
    placement order of the pool (a seeded permutation, or identity)."""
    nb = [-(-int(L) // block_size) for L in context_lens]
    total = sum(nb)
    if pool_blocks < total:
        raise ValueError(f"pool of {pool_blocks} blocks cannot hold {total}")
    if placement == "shuffle":
        order = rng.permutation(pool_blocks)
    elif placement == "identity":
        order = np.arange(pool_blocks)
    else:
        raise ValueError(placement)
    max_nb = max([1] + nb)
    bt = np.full((len(nb), max_nb), -1, dtype=np.int32)
    pos = 0
    for s, n in enumerate(nb):
        bt[s, :n] = order[pos:pos + n]
        pos += n
    return bt


def _token_index(block_tables: np.ndarray, lens: Sequence[int], block_size: int):
    """For every token (sequence-major, then position) its (phys_block, slot)."""
    phys, slot = [], []
    for s, L in enumerate(lens):
        t = np.arange(int(L))
        phys.append(block_tables[s, t // block_size])
        slot.append(t % block_size)
    if not phys:
        return np.zeros(0, np.int64), np.zeros(0, np.int64)
    return np.concatenate(phys).astype(np.int64), np.concatenate(slot).astype(np.int64)


def make_random_case(name: str, num_heads: int, num_kv_heads: int, head_dim: int,
                     block_size: int, context_lens: Sequence[int], dtype: torch.dtype,
                     seed: int, device="cpu", pool_blocks: Optional[int] = None,
                     placement: str = "shuffle", with_append: bool = False,
                     poison: bool = True, partition_size: int = DEFAULT_PARTITION,
                     scale: Optional[float] = None) -> DecodeCase:
    """A decode step over ``len(context_lens)`` sequences with seeded N(0,1) q/K/V.

    With ``with_append`` the last token of every sequence is not in the pool
    yet: its K/V are returned as ``k_new``/``v_new`` with the slot they go to,
    and the decode that follows the append sees the full ``context_lens``.
    """
    lens = np.asarray([int(L) for L in context_lens], dtype=np.int64)
    S = len(lens)
    rng = np.random.default_rng(seed)
    nb_total = int(sum(-(-int(L) // block_size) for L in lens))
    P = int(pool_blocks) if pool_blocks is not None else max(1, nb_total)
    bt = _place_blocks(lens, block_size, P, rng, placement)
    gen = _generator(seed, device)

    q = _randn((S, num_heads, head_dim), gen, dtype, device)
    ntok = int(lens.sum())
    k_tok = _randn((ntok, num_kv_heads, head_dim), gen, dtype, device)
    v_tok = _randn((ntok, num_kv_heads, head_dim), gen, dtype, device)

    fill = float("nan") if poison else 0.0
    k_pool = torch.full((P, num_kv_heads, block_size, head_dim), fill, dtype=dtype, device=device)
    v_pool = torch.full_like(k_pool, fill)

    phys, slot = _token_index(bt, lens, block_size)
    keep = np.ones(ntok, dtype=bool)
    last_idx = np.cumsum(lens) - 1
    k_new = v_new = slot_mapping = None
    if with_append:
        last_idx = last_idx[lens > 0]
        keep[last_idx] = False
        li = torch.as_tensor(last_idx, device=device)
        k_new = k_tok.index_select(0, li).contiguous()
        v_new = v_tok.index_select(0, li).contiguous()
        slots = phys[last_idx] * block_size + slot[last_idx]
        slot_mapping = torch.as_tensor(slots, dtype=torch.int64, device=device)
    kp = torch.as_tensor(phys[keep], device=device)
    ks = torch.as_tensor(slot[keep], device=device)
    kk = torch.as_tensor(np.nonzero(keep)[0], device=device)
    if kp.numel():
        k_pool[kp, :, ks, :] = k_tok.index_select(0, kk)
        v_pool[kp, :, ks, :] = v_tok.index_select(0, kk)
    del k_tok, v_tok

    return DecodeCase(
        name=name, q=q, k_pool=k_pool, v_pool=v_pool,
        block_tables=torch.as_tensor(bt, dtype=torch.int32, device=device),
        context_lens=torch.as_tensor(lens.astype(np.int32), device=device),
        num_heads=num_heads, num_kv_heads=num_kv_heads, head_dim=head_dim,
        block_size=block_size,
        scale=(1.0 / math.sqrt(head_dim)) if scale is None else float(scale),
        partition_size=partition_size, k_new=k_new, v_new=v_new,
        slot_mapping=slot_mapping,
        meta={"seed": seed, "placement": placement, "pool_blocks": P,
              "tokens": ntok, "poison": poison})


def make_sharing_case(name: str, num_heads: int, num_kv_heads: int, head_dim: int,
                      block_size: int, groups, dtype: torch.dtype, seed: int, device="cpu",
                      with_append: bool = False, partition_size: int = DEFAULT_PARTITION,
                      spare_blocks: int = 3) -> DecodeCase:
    """A decode step over groups of sequences that share a prompt's blocks.

    ``groups`` lists ``(prompt_len, own_lens)``: the group's sequences (adjacent
    in the batch) all start with the same ``prompt_len`` tokens, then member
    ``i`` has ``own_lens[i]`` tokens of its own. The prompt's full blocks are
    shared (one physical block, referenced by every member's table, as after
    forking: page "PagedAttention Analysis", section 4). A partly filled last
    prompt block is copied into every member's own first block, as
    copy-on-write leaves it. Placement is a seeded shuffle of the pool; unused
    slots are NaN. With ``with_append`` each sequence's newest token is
    returned as ``k_new``/``v_new`` with its slot (it must be one of the
    member's own tokens).
    """
    B = block_size
    rng = np.random.default_rng(seed)
    gen = _generator(seed, device)
    lens, shared_blocks, own_blocks = [], [], []
    for prompt_len, own in groups:
        nf = prompt_len // B
        shared_blocks.append(nf)
        for o in own:
            L = prompt_len + int(o)
            if with_append and (o < 1):
                raise ValueError("the appended token must be a member's own token")
            lens.append(L)
            own_blocks.append(-(-L // B) - nf)
    P = sum(shared_blocks) + sum(own_blocks) + spare_blocks
    order = rng.permutation(P).tolist()
    S = len(lens)
    bt = np.full((S, max([1] + [-(-L // B) for L in lens])), -1, dtype=np.int32)
    fill = float("nan")
    k_pool = torch.full((P, num_kv_heads, B, head_dim), fill, dtype=dtype, device=device)
    v_pool = torch.full_like(k_pool, fill)
    q = _randn((S, num_heads, head_dim), gen, dtype, device)
    k_new_rows, v_new_rows, slots = [], [], []
    s = 0
    for (prompt_len, own), nf in zip(groups, shared_blocks):
        pk = _randn((prompt_len, num_kv_heads, head_dim), gen, dtype, device)
        pv = _randn((prompt_len, num_kv_heads, head_dim), gen, dtype, device)
        shared = [order.pop() for _ in range(nf)]
        for o in own:
            L = prompt_len + int(o)
            nb = -(-L // B)
            table = shared + [order.pop() for _ in range(nb - nf)]
            bt[s, :nb] = table
            ok = _randn((int(o), num_kv_heads, head_dim), gen, dtype, device)
            ov = _randn((int(o), num_kv_heads, head_dim), gen, dtype, device)
            kt = torch.cat([pk, ok])
            vt = torch.cat([pv, ov])
            t = np.arange(L)
            keep = t < L - 1 if with_append else np.ones(L, dtype=bool)
            ph = torch.as_tensor(np.asarray(table)[t[keep] // B], device=device)
            sl = torch.as_tensor(t[keep] % B, device=device)
            k_pool[ph, :, sl, :] = kt[torch.as_tensor(keep, device=device)]
            v_pool[ph, :, sl, :] = vt[torch.as_tensor(keep, device=device)]
            if with_append:
                k_new_rows.append(kt[L - 1])
                v_new_rows.append(vt[L - 1])
                slots.append(table[(L - 1) // B] * B + (L - 1) % B)
            s += 1
    k_new = v_new = slot_mapping = None
    if with_append:
        k_new = torch.stack(k_new_rows).contiguous()
        v_new = torch.stack(v_new_rows).contiguous()
        slot_mapping = torch.as_tensor(np.asarray(slots, np.int64), device=device)
    return DecodeCase(
        name=name, q=q, k_pool=k_pool, v_pool=v_pool,
        block_tables=torch.as_tensor(bt, dtype=torch.int32, device=device),
        context_lens=torch.as_tensor(np.asarray(lens, np.int32), device=device),
        num_heads=num_heads, num_kv_heads=num_kv_heads, head_dim=head_dim, block_size=B,
        scale=1.0 / math.sqrt(head_dim), partition_size=partition_size, k_new=k_new,
        v_new=v_new, slot_mapping=slot_mapping,
        meta={"seed": seed, "pool_blocks": P, "groups": [(int(pl), [int(o) for o in ow])
                                                         for pl, ow in groups]})


# ---------------------------------------------------------------------------
# The five workloads
# ---------------------------------------------------------------------------

def _lens_tiny(rng):
    return [1, 15, 16, 37]


def _lens_opt13b(rng):
    return rng.integers(128, 2048, size=64, endpoint=True).tolist()


def _lens_llama8b(rng):
    # lognormal around a median of 512 tokens, sigma 1.0, rounded, in [1, 4096]
    x = rng.lognormal(mean=math.log(512.0), sigma=1.0, size=256)
    return np.clip(np.rint(x), 1, 4096).astype(np.int64).tolist()


def _lens_long(rng):
    return rng.integers(32768, 131072, size=8, endpoint=True).tolist()


WORKLOADS = {
    "tiny_f32": dict(num_heads=2, num_kv_heads=2, head_dim=64, block_size=16,
                     dtype="f32", lens=_lens_tiny, pool=lambda nb: 16,
                     partition_size=DEFAULT_PARTITION, seed=388,
                     desc="4 seqs, context_lens {1,15,16,37}, 2 heads MHA, head_dim 64, "
                          "block 16, pool of 16 blocks, fp32"),
    "opt13b_mha_b64": dict(num_heads=40, num_kv_heads=40, head_dim=128, block_size=16,
                           dtype="f16", lens=_lens_opt13b,
                           pool=lambda nb: int(math.ceil(1.2 * nb)),
                           partition_size=DEFAULT_PARTITION, seed=389, append=True,
                           desc="OPT-13B-shaped: 40 heads MHA, head_dim 128, fp16, block 16, "
                                "batch 64, lens U[128,2048], pool 1.2x need, append first"),
    "llama8b_gqa_b256": dict(num_heads=32, num_kv_heads=8, head_dim=128, block_size=16,
                             dtype="bf16", lens=_lens_llama8b, pool=lambda nb: nb,
                             partition_size=DEFAULT_PARTITION, seed=390,
                             desc="Llama-8B-shaped GQA: 32 q heads / 8 kv heads, head_dim 128, "
                                  "bf16, block 16, batch 256, lens lognormal(median 512, "
                                  "sigma 1) in [1,4096]"),
    "long_split_b8": dict(num_heads=32, num_kv_heads=8, head_dim=128, block_size=32,
                          dtype="bf16", lens=_lens_long, pool=lambda nb: nb,
                          partition_size=LONG_CONTEXT_PARTITION, seed=392,
                          desc="long context: batch 8, lens U[32768,131072], 32/8 heads, "
                               "head_dim 128, bf16, block 32, 512-token partitions"),
}


def make_case(workload: str, device="cpu", with_append: Optional[bool] = None,
              seed: Optional[int] = None, num_seqs: Optional[int] = None,
              placement: str = "shuffle", poison: bool = True) -> DecodeCase:
    """Build one of the named workloads (``WORKLOADS``).

    ``num_seqs`` keeps only the first sequences (a bounded sample of the same
    length distribution). The pool then shrinks in proportion.
    """
    w = WORKLOADS[workload]
    sd = w["seed"] if seed is None else int(seed)
    rng = np.random.default_rng(sd)
    lens = w["lens"](rng)
    if num_seqs is not None:
        lens = lens[:num_seqs]
    B = w["block_size"]
    nb = int(sum(-(-int(L) // B) for L in lens))
    pool = w["pool"](nb)
    if num_seqs is not None and workload == "tiny_f32":
        pool = 16
    app = w.get("append", False) if with_append is None else with_append
    case = make_random_case(workload, w["num_heads"], w["num_kv_heads"], w["head_dim"], B,
                            lens, DTYPES[w["dtype"]], seed=sd + 1, device=device,
                            pool_blocks=max(pool, nb), placement=placement,
                            with_append=app, poison=poison,
                            partition_size=w["partition_size"])
    case.meta["desc"] = w["desc"]
    return case


# ---------------------------------------------------------------------------
# Shared prefix / parallel sampling with copy-on-write
# ---------------------------------------------------------------------------

@dataclass
class SharedPrefixCase:
    """Prompts shared by several samples, then per-sample decode steps.

    Built through ``BlockAllocator``: every sample of a prompt references the
    prompt's blocks. The first divergent write into the partly filled last
    prompt block copies it whenever its refcount is above one. The copies
    are ``cow_pairs`` and run before step 0's append.
    """

    k_pool: torch.Tensor
    v_pool: torch.Tensor
    cow_pairs: torch.Tensor          # int32 [N][2] (src, dst)
    steps: List[dict]                # per step: slot_mapping, block_tables, context_lens
    num_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    scale: float
    seed: int
    num_prompts: int
    samples: int
    prompt_len: int
    partition_size: int = DEFAULT_PARTITION
    meta: Dict = field(default_factory=dict)

    @property
    def num_seqs(self) -> int:
        return self.num_prompts * self.samples

    def step_tokens(self, k: int, device=None):
        """Seeded q, k_new, v_new for decode step ``k`` (one token per sequence)."""
        dev = self.k_pool.device if device is None else device
        g = _generator(self.seed * 1000 + 17 + k, dev)
        S, Hq, Hkv, D = self.num_seqs, self.num_heads, self.num_kv_heads, self.head_dim
        dt = self.k_pool.dtype
        q = _randn((S, Hq, D), g, dt, dev)
        kn = _randn((S, Hkv, D), g, dt, dev)
        vn = _randn((S, Hkv, D), g, dt, dev)
        return q, kn, vn


def make_shared_prefix_case(device="cpu", seed: int = 391, num_prompts: int = 16,
                            samples: int = 6, prompt_len: int = 1000,
                            decode_steps: int = 64, num_heads: int = 40,
                            num_kv_heads: int = 40, head_dim: int = 128,
                            block_size: int = 16, dtype=torch.float16,
                            headroom: float = 1.1) -> SharedPrefixCase:
    B = block_size
    prompt_blocks = -(-prompt_len // B)
    final_len = prompt_len + decode_steps
    per_sample_tail = -(-final_len // B) - prompt_blocks + 1  # +1 for the CoW copy
    need = num_prompts * (prompt_blocks + samples * per_sample_tail)
    P = int(math.ceil(headroom * need))
    rng = np.random.default_rng(seed)
    alloc = BlockAllocator(P, B, free_order=rng.permutation(P).tolist())

    gen = _generator(seed, device)
    fill = float("nan")
    k_pool = torch.full((P, num_kv_heads, B, head_dim), fill, dtype=dtype, device=device)
    v_pool = torch.full_like(k_pool, fill)

    seqs = []
    for _ in range(num_prompts):
        root = alloc.new_sequence(prompt_len)
        kt = _randn((prompt_len, num_kv_heads, head_dim), gen, dtype, device)
        vt = _randn((prompt_len, num_kv_heads, head_dim), gen, dtype, device)
        t = np.arange(prompt_len)
        ph = torch.as_tensor(np.asarray(root.table)[t // B], device=device)
        sl = torch.as_tensor(t % B, device=device)
        k_pool[ph, :, sl, :] = kt
        v_pool[ph, :, sl, :] = vt
        forks = [root] + [alloc.fork(root) for _ in range(samples - 1)]
        seqs.extend(forks)

    steps = []
    cow = []
    for k in range(decode_steps):
        slots = []
        for sq in seqs:
            slot, c = alloc.append_slot(sq)
            slots.append(slot)
            if c is not None:
                if k != 0:
                    raise AssertionError("copy-on-write only expected on the first write")
                cow.append((c.src, c.dst))
        max_nb = max(len(sq.table) for sq in seqs)
        bt = np.full((len(seqs), max_nb), -1, dtype=np.int32)
        for i, sq in enumerate(seqs):
            bt[i, :len(sq.table)] = sq.table
        steps.append(dict(
            slot_mapping=torch.as_tensor(np.asarray(slots, np.int64), device=device),
            block_tables=torch.as_tensor(bt, device=device),
            context_lens=torch.as_tensor(np.asarray([sq.num_tokens for sq in seqs], np.int32),
                                         device=device)))
    cow_pairs = torch.as_tensor(np.asarray(cow, np.int32).reshape(-1, 2), device=device)
    return SharedPrefixCase(k_pool=k_pool, v_pool=v_pool, cow_pairs=cow_pairs, steps=steps,
                            num_heads=num_heads, num_kv_heads=num_kv_heads,
                            head_dim=head_dim, block_size=B,
                            scale=1.0 / math.sqrt(head_dim), seed=seed,
                            num_prompts=num_prompts, samples=samples,
                            prompt_len=prompt_len,
                            meta={"pool_blocks": P, "copies": len(cow)})


def make_beam_search_case(device="cpu", seed: int = 393, num_requests: int = 32, width: int = 4,
                          prompt_len: int = 512, steps: int = 127, num_heads: int = 32,
                          num_kv_heads: int = 8, head_dim: int = 128, block_size: int = 16,
                          dtype=torch.bfloat16, partition_size: int = DEFAULT_PARTITION):
    """Beam search over ``num_requests`` requests of ``width`` beams (page
    "PagedAttention Analysis", section 4: the beams share the prompt and
    intermediate blocks, and the sharing changes every step).

    Every step each request's new beams continue seeded random parents; the
    copy-on-write block copies and the new tokens' K/V (N(0,1)) are applied to
    the pools. After ``steps`` steps, the returned case is the next step: its
    copies already applied, ``k_new``/``v_new``/``slot_mapping`` the tokens it
    appends, and ``context_lens`` counting them. Sharing statistics are in
    ``meta``: the blocks the beams hold, the blocks they would hold unshared.
    """
    B = block_size
    rng = np.random.default_rng(seed)
    gen = _generator(seed, device)
    per_req = width * (-(-(prompt_len + steps + 1) // B) + 1)  # bound without sharing
    P = num_requests * per_req
    alloc = BlockAllocator(P, B, free_order=rng.permutation(P).tolist())
    fill = float("nan")
    k_pool = torch.full((P, num_kv_heads, B, head_dim), fill, dtype=dtype, device=device)
    v_pool = torch.full_like(k_pool, fill)

    def write(slots, kt, vt):
        s = np.asarray(slots, np.int64)
        ph = torch.as_tensor(s // B, device=device)
        sl = torch.as_tensor(s % B, device=device)
        k_pool[ph, :, sl, :] = kt
        v_pool[ph, :, sl, :] = vt

    def copy(copies):
        if copies:
            src = torch.as_tensor([c.src for c in copies], device=device)
            dst = torch.as_tensor([c.dst for c in copies], device=device)
            k_pool[dst] = k_pool[src]
            v_pool[dst] = v_pool[src]

    searches = []
    for _ in range(num_requests):
        bs = BeamSearch(alloc, prompt_len, width)
        t = np.arange(prompt_len)
        write(np.asarray(bs.beams[0].table)[t // B] * B + t % B,
              _randn((prompt_len, num_kv_heads, head_dim), gen, dtype, device),
              _randn((prompt_len, num_kv_heads, head_dim), gen, dtype, device))
        searches.append(bs)

    def one_step():
        slots, copies = [], []
        for bs in searches:
            s, c = bs.step(rng.integers(0, width, size=width))
            slots += s
            copies += c
        copy(copies)
        return slots, len(copies)

    for _ in range(steps):
        slots, _ = one_step()
        n = len(slots)
        write(slots, _randn((n, num_kv_heads, head_dim), gen, dtype, device),
              _randn((n, num_kv_heads, head_dim), gen, dtype, device))
    slots, ncopies = one_step()
    beams = [b for bs in searches for b in bs.beams]
    S = len(beams)
    max_nb = max(len(b.table) for b in beams)
    bt = np.full((S, max_nb), -1, dtype=np.int32)
    for i, b in enumerate(beams):
        bt[i, :len(b.table)] = b.table
    q = _randn((S, num_heads, head_dim), gen, dtype, device)
    k_new = _randn((S, num_kv_heads, head_dim), gen, dtype, device)
    v_new = _randn((S, num_kv_heads, head_dim), gen, dtype, device)
    in_use = sum(bs.blocks_in_use() for bs in searches)
    unshared = sum(bs.blocks_unshared() for bs in searches)
    return DecodeCase(
        name="beam_search", q=q, k_pool=k_pool, v_pool=v_pool,
        block_tables=torch.as_tensor(bt, device=device),
        context_lens=torch.as_tensor(np.asarray([b.num_tokens for b in beams], np.int32),
                                     device=device),
        num_heads=num_heads, num_kv_heads=num_kv_heads, head_dim=head_dim, block_size=B,
        scale=1.0 / math.sqrt(head_dim), partition_size=partition_size, k_new=k_new,
        v_new=v_new, slot_mapping=torch.as_tensor(np.asarray(slots, np.int64), device=device),
        meta={"seed": seed, "pool_blocks": P, "requests": num_requests, "width": width,
              "blocks_in_use": in_use, "blocks_unshared": unshared,
              "copies_last_step": ncopies, "allocator": alloc, "searches": searches})


def make_prefix_cache_case(device="cpu", seed: int = 394, num_requests: int = 64,
                           system_len: int = 1024, groups: int = 8, group_len: int = 512,
                           suffix_range=(128, 256), num_heads: int = 32, num_kv_heads: int = 8,
                           head_dim: int = 128, block_size: int = 16, dtype=torch.bfloat16,
                           partition_size: int = DEFAULT_PARTITION):
    """Automatic prefix caching (page "PagedAttention Analysis", section 4):
    requests built from synthetic token ids (a system prompt shared by all, a
    prefix shared within each of ``groups`` groups, a unique suffix) get their
    blocks from a PrefixCache. Each block that misses the cache is filled with
    N(0,1) K/V when it is first allocated; hits read what was written then.
    The total length of a request is never a multiple of the block size, and its
    last token is the one the step appends (``k_new``/``v_new``/``slot_mapping``),
    so the appended token always lands in the request's private last block.
    Cache statistics are in ``meta``."""
    B = block_size
    rng = np.random.default_rng(seed)
    gen = _generator(seed, device)
    system = rng.integers(0, 32000, size=system_len).tolist()
    group_prefix = [rng.integers(0, 32000, size=group_len).tolist() for _ in range(groups)]
    reqs = []
    for r in range(num_requests):
        n = int(rng.integers(suffix_range[0], suffix_range[1] + 1))
        total = system_len + group_len + n
        if total % B == 0:
            n += 1
        reqs.append(system + group_prefix[r % groups] + rng.integers(0, 32000, size=n).tolist())
    P = sum(-(-len(t) // B) for t in reqs)  # enough without any sharing
    alloc = BlockAllocator(P, B, free_order=rng.permutation(P).tolist())
    cache = PrefixCache(alloc)
    fill = float("nan")
    k_pool = torch.full((P, num_kv_heads, B, head_dim), fill, dtype=dtype, device=device)
    v_pool = torch.full_like(k_pool, fill)
    seqs = []
    for toks in reqs:
        sq, fills = cache.new_sequence(toks)
        L = len(toks)
        for j in fills:
            n = min(B, L - 1 - j * B)  # the last token is appended by the step itself
            if n <= 0:
                continue
            blk = sq.table[j]
            k_pool[blk, :, :n, :] = _randn((num_kv_heads, n, head_dim), gen, dtype, device)
            v_pool[blk, :, :n, :] = _randn((num_kv_heads, n, head_dim), gen, dtype, device)
        seqs.append(sq)
    S = len(seqs)
    max_nb = max(len(sq.table) for sq in seqs)
    bt = np.full((S, max_nb), -1, dtype=np.int32)
    for i, sq in enumerate(seqs):
        bt[i, :len(sq.table)] = sq.table
    lens = np.asarray([sq.num_tokens for sq in seqs], np.int32)
    slots = np.asarray([sq.table[(L - 1) // B] * B + (L - 1) % B for sq, L in zip(seqs, lens)],
                       np.int64)
    q = _randn((S, num_heads, head_dim), gen, dtype, device)
    k_new = _randn((S, num_kv_heads, head_dim), gen, dtype, device)
    v_new = _randn((S, num_kv_heads, head_dim), gen, dtype, device)
    in_use = len({b for sq in seqs for b in sq.table})
    return DecodeCase(
        name="prefix_cache", q=q, k_pool=k_pool, v_pool=v_pool,
        block_tables=torch.as_tensor(bt, device=device),
        context_lens=torch.as_tensor(lens, device=device),
        num_heads=num_heads, num_kv_heads=num_kv_heads, head_dim=head_dim, block_size=B,
        scale=1.0 / math.sqrt(head_dim), partition_size=partition_size, k_new=k_new,
        v_new=v_new, slot_mapping=torch.as_tensor(slots, device=device),
        meta={"seed": seed, "pool_blocks": P, "hits": cache.hits, "misses": cache.misses,
              "blocks_in_use": in_use, "blocks_unshared": int(sum(len(sq.table) for sq in seqs)),
              "tokens": [list(t) for t in reqs], "cache": cache})
