"""Random operation sequences on the host block bookkeeping (CPU).

Page "추론 엔진에서의 메모리 가상화" (copy-on-write section) and page
"PagedAttention Analysis" (sections 4 and 6) describe a refcounted block
allocator: forks share blocks, a write into a shared block copies it first,
and preempted groups of sequences are swapped to a CPU block pool and back,
all or nothing. A state machine drives random new / fork / append / release /
swap-out / swap-in steps over a tiny pool and, after every step, checks:

* refcounts: every block's count equals the table entries that point at it,
  on its own side (GPU pool or swap space), and the free lists hold exactly
  the unreferenced blocks;
* tables: ceil(num_tokens / B) entries per sequence;
* contents: the block copies and moves the allocator returns, applied to a
  simulated pool of token ids, keep every sequence's logical tokens intact.

A second machine does the same for the prefix cache (page "PagedAttention
Analysis", section 4: blocks keyed by a hash of the whole prefix, shared
through a global table): requests over a two-letter alphabet collide often,
and every cache hit must serve a block that holds exactly the requested
tokens, also after cached blocks were released, evicted and reused.

Beam search (section 4 of the same page: the beams share the prompt and
intermediate blocks, and the sharing changes every step) is checked the same
way: with random parents every step, each beam must read back its parent's
tokens plus its own new one once the step's copies have run before its
writes, and releasing the request must free every block.
"""

from collections import Counter

from hypothesis import given, settings
from hypothesis import strategies as st
from hypothesis.stateful import RuleBasedStateMachine, invariant, precondition, rule

from pkv_inputs import BeamSearch, BlockAllocator, PrefixCache, SwapSpace

P, B = 24, 4


class BlockBookkeeping(RuleBasedStateMachine):
    def __init__(self):
        super().__init__()
        self.gpu = BlockAllocator(P, B, free_order=list(range(P))[::-1])
        self.swap = SwapSpace(self.gpu)
        # simulated contents: (side, block) -> list of B token ids (None = unwritten)
        self.data = {}
        self.seqs = []      # live SeqStates
        self.tokens = []    # the logical tokens each live sequence must read back
        self.next_tok = 0

    # -- helpers ---------------------------------------------------------------
    def _side(self, seq):
        return "cpu" if seq.on_host else "gpu"

    def _block(self, side, b):
        return self.data.setdefault((side, b), [None] * B)

    def _write(self, seq, slot, tok):
        self._block(self._side(seq), slot // B)[slot % B] = tok

    def _gpu_idx(self):
        return [i for i, s in enumerate(self.seqs) if not s.on_host]

    def _host_idx(self):
        return [i for i, s in enumerate(self.seqs) if s.on_host]

    def _fresh(self, n):
        toks = list(range(self.next_tok, self.next_tok + n))
        self.next_tok += n
        return toks

    # -- rules -----------------------------------------------------------------
    @rule(n=st.integers(1, 9))
    def new_sequence(self, n):
        if self.gpu.num_free < -(-n // B):
            return
        seq = self.gpu.new_sequence(n)
        toks = self._fresh(n)
        for t, tok in enumerate(toks):
            self._write(seq, seq.table[t // B] * B + t % B, tok)
        self.seqs.append(seq)
        self.tokens.append(toks)

    @precondition(lambda self: any(not s.on_host for s in self.seqs))
    @rule(pick=st.integers(0, 10 ** 6))
    def fork(self, pick):
        idx = self._gpu_idx()
        i = idx[pick % len(idx)]
        self.seqs.append(self.gpu.fork(self.seqs[i]))
        self.tokens.append(list(self.tokens[i]))

    @precondition(lambda self: any(not s.on_host for s in self.seqs))
    @rule(pick=st.integers(0, 10 ** 6))
    def append(self, pick):
        if self.gpu.num_free < 1:
            return
        idx = self._gpu_idx()
        i = idx[pick % len(idx)]
        seq = self.seqs[i]
        slot, cow = self.gpu.append_slot(seq)
        if cow is not None:  # the copy runs before the write
            self.data[("gpu", cow.dst)] = list(self._block("gpu", cow.src))
        tok = self._fresh(1)[0]
        self._write(seq, slot, tok)
        self.tokens[i].append(tok)

    @precondition(lambda self: any(not s.on_host for s in self.seqs))
    @rule(pick=st.integers(0, 10 ** 6))
    def release(self, pick):
        idx = self._gpu_idx()
        i = idx[pick % len(idx)]
        self.gpu.release(self.seqs[i])
        del self.seqs[i], self.tokens[i]

    @precondition(lambda self: any(not s.on_host for s in self.seqs))
    @rule(mask=st.integers(1, 2 ** 12))
    def swap_out(self, mask):
        idx = self._gpu_idx()
        group = [self.seqs[i] for k, i in enumerate(idx) if (mask >> (k % 12)) & 1] or \
            [self.seqs[idx[0]]]
        before = [(list(s.table), s.on_host) for s in group]
        try:
            moves = self.swap.swap_out(group)
        except MemoryError:  # all or nothing: the group is untouched
            assert [(list(s.table), s.on_host) for s in group] == before
            return
        for m in moves:
            self.data[("cpu", m.dst)] = list(self._block("gpu", m.src))

    @precondition(lambda self: any(s.on_host for s in self.seqs))
    @rule(mask=st.integers(1, 2 ** 12))
    def swap_in(self, mask):
        idx = self._host_idx()
        group = [self.seqs[i] for k, i in enumerate(idx) if (mask >> (k % 12)) & 1] or \
            [self.seqs[idx[0]]]
        before = [(list(s.table), s.on_host) for s in group]
        try:
            moves = self.swap.swap_in(group)
        except MemoryError:
            assert [(list(s.table), s.on_host) for s in group] == before
            return
        for m in moves:
            self.data[("gpu", m.dst)] = list(self._block("cpu", m.src))

    # -- invariants ------------------------------------------------------------
    @invariant()
    def refcounts_and_free_lists(self):
        for alloc, on_host in ((self.gpu, False), (self.swap.cpu, True)):
            refs = Counter(b for s in self.seqs if s.on_host == on_host for b in s.table)
            for b in range(alloc.num_blocks):
                assert alloc.refcount(b) == refs.get(b, 0), (on_host, b)
            assert alloc.num_free == alloc.num_blocks - len(refs)

    @invariant()
    def tables_and_contents(self):
        for seq, toks in zip(self.seqs, self.tokens):
            assert seq.num_tokens == len(toks)
            assert len(seq.table) == -(-seq.num_tokens // B)
            side = self._side(seq)
            got = [self._block(side, seq.table[t // B])[t % B] for t in range(seq.num_tokens)]
            assert got == toks


TestBlockBookkeeping = BlockBookkeeping.TestCase
TestBlockBookkeeping.settings = settings(max_examples=150, stateful_step_count=40, deadline=None)


class PrefixCacheBookkeeping(RuleBasedStateMachine):
    def __init__(self):
        super().__init__()
        self.alloc = BlockAllocator(16, B, free_order=list(range(16))[::-1])
        self.cache = PrefixCache(self.alloc)
        self.data = {}   # block -> the B tokens written into it
        self.seqs = []
        self.tokens = []

    @rule(toks=st.lists(st.integers(0, 1), min_size=1, max_size=14))
    def request(self, toks):
        nb = -(-len(toks) // B)
        if self.alloc.num_free < nb:
            return
        hits0 = self.cache.hits
        seq, fills = self.cache.new_sequence(toks)
        assert len(seq.table) == nb
        full = len(toks) // B
        for j, b in enumerate(seq.table):
            want = toks[j * B:(j + 1) * B]
            if j in fills:
                self.data[b] = list(want)          # the caller fills misses and the tail
            else:
                assert j < full                     # only full blocks are shared
                assert self.data.get(b) == want     # a hit holds exactly these tokens
        assert self.cache.hits - hits0 == nb - len(fills)
        self.seqs.append(seq)
        self.tokens.append(list(toks))

    @precondition(lambda self: self.seqs)
    @rule(pick=st.integers(0, 10 ** 6))
    def release(self, pick):
        i = pick % len(self.seqs)
        self.cache.release(self.seqs[i])
        del self.seqs[i], self.tokens[i]

    @invariant()
    def refcounts_keys_and_contents(self):
        refs = Counter(b for s in self.seqs for b in s.table)
        for b in range(self.alloc.num_blocks):
            assert self.alloc.refcount(b) == refs.get(b, 0), b
        assert self.alloc.num_free == self.alloc.num_blocks - len(refs)
        assert {b: k for k, b in self.cache.table.items()} == self.cache.key_of
        for seq, toks in zip(self.seqs, self.tokens):
            got = [self.data[seq.table[t // B]][t % B] for t in range(len(toks))]
            assert got == toks


TestPrefixCacheBookkeeping = PrefixCacheBookkeeping.TestCase
TestPrefixCacheBookkeeping.settings = settings(max_examples=150, stateful_step_count=40,
                                               deadline=None)


@settings(max_examples=200, deadline=None)
@given(width=st.integers(1, 4), prompt=st.integers(1, 10),
       parents=st.lists(st.lists(st.integers(0, 3), min_size=4, max_size=4), max_size=12))
def test_beam_search_contents_and_no_leaks(width, prompt, parents):
    P_beam = width * (-(-(prompt + len(parents)) // B) + 1)
    alloc = BlockAllocator(P_beam, B, free_order=list(range(P_beam))[::-1])
    bs = BeamSearch(alloc, prompt, width)
    data = {}
    root = bs.beams[0]
    toks = [list(range(prompt)) for _ in range(width)]
    for t in range(prompt):
        data.setdefault(root.table[t // B], [None] * B)[t % B] = t
    nxt = prompt
    for step, ps in enumerate(parents):
        ps = [p % width for p in ps[:width]]
        slots, copies = bs.step(ps)
        for cp in copies:  # every copy runs before any of the step's writes
            data[cp.dst] = list(data[cp.src])
        toks = [toks[p] + [nxt + i] for i, p in enumerate(ps)]
        for i, slot in enumerate(slots):
            data.setdefault(slot // B, [None] * B)[slot % B] = nxt + i
        nxt += width
        for beam, want in zip(bs.beams, toks):
            assert beam.num_tokens == len(want)
            got = [data[beam.table[t // B]][t % B] for t in range(beam.num_tokens)]
            assert got == want, f"step {step}"
    bs.release()
    assert alloc.num_free == P_beam
