"""The C-ABI library on a host without a GPU: it builds, loads, exports every
function ``include/pkv.h`` declares, and its synchronous argument checks
return the documented status codes. Only calls rejected before any launch are
made here."""

import ctypes
import os
import re

import pytest

import paged_kv_cache_387_b200 as pkv
from paged_kv_cache_387_b200 import build as pkv_build

HEADER_DIR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include")


def declared_functions():
    names = []
    for fn in sorted(os.listdir(HEADER_DIR)):
        if not fn.endswith(".h"):
            continue
        text = open(os.path.join(HEADER_DIR, fn)).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"^[A-Za-z_][\w \*]*?\b([A-Za-z_]\w*)\s*\(", text, flags=re.M):
            line = m.group(0)
            if line.startswith(("typedef", "#", "enum", "return")):
                continue
            names.append(m.group(1))
    return names


@pytest.fixture(scope="module")
def lib():
    pkv_build.build()
    return pkv.load_library()


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert set(pkv.EXPORTS) <= set(names), names
    raw = ctypes.CDLL(pkv.LIB_PATH)
    for n in names:
        assert hasattr(raw, n), f"{n} declared in include/ but not exported"


def test_status_strings(lib):
    assert lib.pkv_status_string(0) == b"ok"
    assert lib.pkv_status_string(-1) == b"invalid argument"
    assert lib.pkv_status_string(-2) == b"unsupported configuration"
    assert lib.pkv_status_string(-3) == b"CUDA error"


def test_workspace_arithmetic(lib):
    f = lib.pkv_decode_workspace_bytes
    rnd = lambda x: -(-x // 256) * 256

    def expected(S, Hq, D, L, P):
        parts = 1 if P == 0 else -(-max(L, 1) // P)  # partitions of the longest context
        total = 256 + rnd(S * parts * 8) + rnd(2 * S * 4)  # sched words, work list, group words
        pieces = min(512, S * Hq * parts)                    # tail split: counters, 8 rows each
        total += rnd(pieces * 4) + rnd(pieces * 8 * D * 4) + rnd(pieces * 8 * 4)
        if parts > 1:
            chunks = -(-parts // 16)
            total += (rnd(S * Hq * chunks * 4) + rnd(S * Hq * 4)      # merge counters
                      + rnd(S * Hq * parts * D * 4) + rnd(S * Hq * parts * 4))  # partials
            if chunks > 1:                                             # chunk results
                total += rnd(S * Hq * chunks * D * 4) + rnd(S * Hq * chunks * 4)
        return total

    # tail-split region: min(512, S*Hq*partitions) pieces, each a counter, 8
    # fp32 output rows and 8 fp32 log2-sum-exp values
    def tail(S, Hq, D, parts):
        n = min(512, S * Hq * parts)
        return rnd(n * 4) + rnd(n * 8 * D * 4) + rnd(n * 8 * 4)

    assert tail(8, 32, 128, 1) == 1024 + 256 * 8 * 128 * 4 + 256 * 8 * 4
    assert tail(100, 8, 64, 1) == 2048 + 512 * 8 * 64 * 4 + 512 * 8 * 4  # capped at 512
    # scheduling words (256 B) + work list (8 bytes per (seq, partition)) +
    # shared-prefix group words (two int32 per sequence), each region rounded
    # up to 256 B
    assert f(8, 32, 128, 512, 512) == 256 + 256 + 256 + tail(8, 32, 128, 1)  # no partials
    assert f(8, 32, 128, 100, 0) == 256 + 256 + 256 + tail(8, 32, 128, 1)    # unsplit
    assert f(100, 8, 64, 100, 0) == 256 + rnd(100 * 8) + rnd(100 * 8) + tail(100, 8, 64, 1)
    # 8 seqs x 32 heads x 256 partitions (16 merge chunks of 16): chunk and
    # final merge counters, fp32 partition outputs + lse, chunk results + lse
    S, Hq, D, P, C = 8, 32, 128, 256, 16
    assert f(S, Hq, D, 131072, 512) == (256 + S * P * 8 + 256 + tail(S, Hq, D, P)
                                        + S * Hq * C * 4 + S * Hq * 4
                                        + S * Hq * P * D * 4 + S * Hq * P * 4
                                        + S * Hq * C * D * 4 + S * Hq * C * 4)
    # 33 tokens in 16-token partitions = 3 partitions, one merge chunk
    assert f(1, 1, 64, 33, 16) == (256 + 256 + 256 + tail(1, 1, 64, 3)
                                   + 256 + 256 + 3 * 64 * 4 + 256)
    for args in [(100, 8, 64, 100, 0), (3, 40, 128, 1064, 2048), (256, 32, 128, 4096, 2048),
                 (5, 2, 64, 20000, 16)]:
        assert f(*args) == expected(*args), args
    assert f(0, 32, 128, 512, 512) == 0


def test_auto_partition_rule(lib):
    r = lib.pkv_resolve_partition
    AUTO = pkv.PARTITION_AUTO
    # explicit sizes pass through
    assert r(1, 32, 4096, 512) == 512 and r(1, 32, 4096, 0) == 0
    # big batches: 2048-token partitions (one partition when the contexts are shorter)
    assert r(256, 32, 4096, AUTO) == 2048
    assert r(64, 40, 2048, AUTO) == 2048
    assert r(256, 32, 100, AUTO) == 256
    # small batches: about 1024 (sequence, partition, head) rows, partitions >= 256 tokens
    assert r(1, 32, 4096, AUTO) == 256       # n = 32 -> 128 tokens -> raised to 256
    assert r(1, 32, 32768, AUTO) == 1024     # n = 32 -> 1024
    assert r(1, 32, 131072, AUTO) == 2048    # n = 32 -> 4096 -> lowered to 2048
    assert r(2, 32, 20000, AUTO) == 1264     # n = 16 -> 1250 -> multiple of 16
    assert r(4, 32, 16384, AUTO) == 2048     # n = 8 -> 2048
    assert r(8, 8, 3000, AUTO) == 256        # n = 16 -> 188 -> 256
    assert r(0, 32, 0, AUTO) == 256          # degenerate shapes stay valid
    for S, Hq, L in [(1, 32, 4096), (3, 8, 70000), (256, 32, 4096), (5, 40, 2000)]:
        assert r(S, Hq, L, AUTO) % 16 == 0
        assert (lib.pkv_decode_workspace_bytes(S, Hq, 128, L, AUTO)
                == lib.pkv_decode_workspace_bytes(S, Hq, 128, L, r(S, Hq, L, AUTO)))
    assert pkv.resolve_partition(1, 32, 4096) == 256  # the binding's default is AUTO


FAKE = ctypes.c_void_p(0x10000)  # never dereferenced: every call below is rejected first


def decode(lib, **kw):
    args = dict(out=FAKE, q=FAKE, k=FAKE, v=FAKE, bt=FAKE, cl=FAKE, S=2, Hq=8, Hkv=2, D=128,
                B=16, MB=4, P=10, L=64, scale=0.088, dtype=2, part=512, ws=None, wsb=0,
                err=None, stream=None)
    args.update(kw)
    return lib.paged_attn_decode(*args.values())


def test_decode_argument_checks(lib):
    assert decode(lib, out=None) == pkv.PKV_EINVAL
    assert decode(lib, Hq=6, Hkv=4) == pkv.PKV_EINVAL
    assert decode(lib, part=24) == pkv.PKV_EINVAL
    assert decode(lib, part=-2) == pkv.PKV_EINVAL                     # only -1 means AUTO
    assert decode(lib, part=pkv.PARTITION_AUTO, L=200000, ws=None, wsb=0) == pkv.PKV_EINVAL
    assert decode(lib, dtype=7) == pkv.PKV_EINVAL
    assert decode(lib, scale=float("nan")) == pkv.PKV_EINVAL
    assert decode(lib, L=2048, ws=None, wsb=0) == pkv.PKV_EINVAL     # workspace needed
    assert decode(lib, D=96) == pkv.PKV_EUNSUPPORTED
    assert decode(lib, B=12) == pkv.PKV_EUNSUPPORTED                  # 16-bit needs B % 8 == 0
    assert decode(lib, B=264) == pkv.PKV_EUNSUPPORTED                 # and B <= 256
    assert decode(lib, Hq=32, Hkv=2) == pkv.PKV_EUNSUPPORTED          # group of 16 > 8
    assert decode(lib, q=ctypes.c_void_p(0x10008)) == pkv.PKV_EINVAL  # misaligned
    assert decode(lib, S=0) == pkv.PKV_OK                             # nothing to do


def test_append_and_copy_argument_checks(lib):
    ap = lib.kv_cache_append
    assert ap(FAKE, FAKE, FAKE, FAKE, None, 4, 2, 128, 16, 10, 1, None, None) == pkv.PKV_EINVAL
    assert ap(FAKE, FAKE, FAKE, FAKE, FAKE, 4, 2, 4, 16, 10, 1, None, None) == pkv.PKV_EUNSUPPORTED
    assert ap(FAKE, FAKE, FAKE, FAKE, FAKE, 0, 2, 128, 16, 10, 1, None, None) == pkv.PKV_OK
    cp = lib.kv_block_copy
    assert cp(FAKE, None, FAKE, 3, 2, 128, 16, 10, 1, None, None) == pkv.PKV_EINVAL
    assert cp(FAKE, FAKE, FAKE, -1, 2, 128, 16, 10, 1, None, None) == pkv.PKV_EINVAL
    assert cp(FAKE, FAKE, None, 0, 2, 128, 16, 10, 1, None, None) == pkv.PKV_OK


@pytest.mark.gpu
def test_binding_refuses_cpu_tensors(lib):
    """A device `out` with q (or the pools) left on the host: the binding
    refuses the host input before anything reaches the library."""
    import torch
    x = torch.zeros(2, 8, 128, dtype=torch.bfloat16)
    k = torch.zeros(4, 2, 16, 128, dtype=torch.bfloat16)
    bt = torch.zeros(2, 1, dtype=torch.int32)
    out = torch.empty(2, 8, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ValueError, match="q must be a CUDA tensor"):
        pkv.paged_attn_decode(out, x, k.cuda(), k.cuda(), bt.cuda(), bt[:, 0].cuda(), 0.1, 16)
    with pytest.raises(ValueError, match="k_pool must be a CUDA tensor"):
        pkv.paged_attn_decode(out, x.cuda(), k, k, bt.cuda(), bt[:, 0].cuda(), 0.1, 16)


def test_binding_refuses_host_q(lib):
    """q on the host is refused before anything reaches the library (no GPU needed)."""
    import torch
    x = torch.zeros(2, 8, 128, dtype=torch.bfloat16)
    k = torch.zeros(4, 2, 16, 128, dtype=torch.bfloat16)
    bt = torch.zeros(2, 1, dtype=torch.int32)
    with pytest.raises(ValueError, match="q must be a CUDA tensor"):
        pkv.paged_attn_decode(x.clone(), x, k, k, bt, bt[:, 0].contiguous(), 0.1, 16)


@pytest.mark.gpu
def test_binding_refuses_unpinned_host_output(lib):
    """A host `out` is accepted only when it is page-locked."""
    import torch
    x = torch.zeros(2, 8, 128, dtype=torch.bfloat16, device="cuda")
    k = torch.zeros(4, 2, 16, 128, dtype=torch.bfloat16, device="cuda")
    bt = torch.zeros(2, 1, dtype=torch.int32, device="cuda")
    out = torch.zeros(2, 8, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="pinned"):
        pkv.paged_attn_decode(out, x, k, k, bt, bt[:, 0].contiguous(), 0.1, 16)


def test_wait_timeout_check_arguments(lib):
    f = lib.pkv_check_wait_timeout
    assert f(0, FAKE, None) == pkv.PKV_EINVAL           # limit must be positive
    assert f(5_000_000_000, FAKE, None) == pkv.PKV_EINVAL
    assert f(1000, None, None) == pkv.PKV_EINVAL         # err is required
