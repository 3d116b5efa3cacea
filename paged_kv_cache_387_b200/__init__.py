"""Python binding of the paged KV-cache decode library (``libpkv.so``).

The functions below only marshal arguments: they check torch tensors' devices,
dtypes, shapes and contiguity, pass their device pointers and the current CUDA
stream to the C ABI declared in ``include/pkv.h``, and raise on a non-zero
status. Every step of the computation runs in the library's CUDA kernels;
there is no fallback path. If the library is not built, every call raises.

Pool layout: ``[num_blocks][num_kv_heads][block_size][head_dim]``, head_dim
contiguous; token t of a sequence is at block ``block_tables[s][t // B]``,
slot ``t % B``.
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libpkv.so")

PKV_OK, PKV_EINVAL, PKV_EUNSUPPORTED, PKV_ECUDA = 0, -1, -2, -3
DEV_ERRORS = {1: "block id out of range", 2: "append slot out of range",
              3: "copy or swap pair out of range", 4: "context length above max_context_len",
              5: "copy wait timed out"}
DTYPE_CODES = {torch.float32: 0, torch.float16: 1, torch.bfloat16: 2}
PARTITION_AUTO = -1  # the library picks the partition length from the batch shape
DEFAULT_PARTITION = PARTITION_AUTO
# Decode kernel selection (pkv_set_decode_dispatch): the single-wave kernel for
# calls that fit one wave of CTAs, else the persistent kernel.
DISPATCH_AUTO, DISPATCH_PERSISTENT, DISPATCH_WAVE_CTA, DISPATCH_WAVE_WARP = 0, 1, 2, 3
DISPATCH_WAVE_CTA8 = 4

EXPORTS = ("paged_attn_decode", "paged_attn_decode_append", "kv_cache_append",
           "kv_block_copy", "kv_block_swap", "pkv_check_wait_timeout",
           "pkv_decode_workspace_bytes", "pkv_resolve_partition", "pkv_set_decode_dispatch",
           "pkv_status_string")


class PkvError(RuntimeError):
    def __init__(self, fn: str, status: int, msg: str):
        super().__init__(f"{fn}: {msg} (status {status})")
        self.status = status


_lib = None


def load_library():
    """Load ``libpkv.so`` (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            f"CUDA library not built: {LIB_PATH} is missing "
            "(run `python paged_kv_cache_387_b200/build.py`)")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, F, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    lib.paged_attn_decode.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, I, I, F, I, I, P, Z, P, P]
    lib.paged_attn_decode.restype = I
    lib.paged_attn_decode_append.argtypes = [P, P, P, P, P, P, P, P, I, I, I, I, I, I, I, I, F,
                                             I, I, P, Z, P, P]
    lib.paged_attn_decode_append.restype = I
    lib.kv_cache_append.argtypes = [P, P, P, P, P, I, I, I, I, I, I, P, P]
    lib.kv_cache_append.restype = I
    lib.kv_block_copy.argtypes = [P, P, P, I, I, I, I, I, I, P, P]
    lib.kv_block_copy.restype = I
    lib.kv_block_swap.argtypes = [P, P, P, P, P, I, I, I, I, I, I, I, P, P]
    lib.kv_block_swap.restype = I
    lib.pkv_check_wait_timeout.argtypes = [ctypes.c_longlong, P, P]
    lib.pkv_check_wait_timeout.restype = I
    lib.pkv_decode_workspace_bytes.argtypes = [I, I, I, I, I]
    lib.pkv_decode_workspace_bytes.restype = Z
    lib.pkv_resolve_partition.argtypes = [I, I, I, I]
    lib.pkv_resolve_partition.restype = I
    lib.pkv_set_decode_dispatch.argtypes = [I]
    lib.pkv_set_decode_dispatch.restype = I
    lib.pkv_status_string.argtypes = [I]
    lib.pkv_status_string.restype = ctypes.c_char_p
    _lib = lib
    return lib


def _check(fn: str, rc: int):
    if rc != PKV_OK:
        msg = load_library().pkv_status_string(rc).decode()
        raise PkvError(fn, rc, msg)


def _dev_ptr(t: Optional[torch.Tensor], name: str, device=None):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor) or t.device.type != "cuda":
        raise ValueError(f"{name} must be a CUDA tensor")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _out_ptr(t: torch.Tensor, device):
    """`out` of a decode call: a CUDA tensor on `device`, or a page-locked
    (pinned) host tensor, which the kernels write directly over the bus."""
    if isinstance(t, torch.Tensor) and t.device.type == "cpu":
        if not t.is_pinned():
            raise ValueError("out on the host must be pinned (page-locked) memory")
        if not t.is_contiguous():
            raise ValueError("out must be contiguous")
        return ctypes.c_void_p(t.data_ptr())
    return _dev_ptr(t, "out", device)


def _stream_ptr(stream, device):
    s = torch.cuda.current_stream(device) if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def decode_workspace_bytes(num_seqs: int, num_heads: int, head_dim: int, max_context_len: int,
                           partition_size: int = DEFAULT_PARTITION) -> int:
    return int(load_library().pkv_decode_workspace_bytes(num_seqs, num_heads, head_dim,
                                                         max_context_len, partition_size))


def resolve_partition(num_seqs: int, num_heads: int, max_context_len: int,
                      partition_size: int = DEFAULT_PARTITION) -> int:
    """The partition length a decode call uses (``PARTITION_AUTO`` resolved)."""
    return int(load_library().pkv_resolve_partition(num_seqs, num_heads, max_context_len,
                                                    partition_size))


def set_decode_dispatch(mode: int) -> int:
    """Select the decode kernel for fp16 / bf16 calls, process-wide
    (``DISPATCH_*``); returns the previous mode."""
    rc = int(load_library().pkv_set_decode_dispatch(int(mode)))
    if rc < 0:
        _check("pkv_set_decode_dispatch", rc)
    return rc


def paged_attn_decode(out: torch.Tensor, q: torch.Tensor, k_pool: torch.Tensor,
                      v_pool: torch.Tensor, block_tables: torch.Tensor,
                      context_lens: torch.Tensor, scale: float, max_context_len: int,
                      partition_size: int = DEFAULT_PARTITION,
                      workspace: Optional[torch.Tensor] = None,
                      err: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """One decode step of paged attention; writes ``out`` [S][Hq][D]."""
    lib = load_library()
    _dev_ptr(q, "q")  # q decides the device every other tensor must be on
    dev = q.device
    if q.dtype not in DTYPE_CODES or out.dtype != q.dtype or k_pool.dtype != q.dtype \
            or v_pool.dtype != q.dtype:
        raise TypeError("q, out, k_pool and v_pool must share one of float32/float16/bfloat16")
    if block_tables.dtype != torch.int32 or context_lens.dtype != torch.int32:
        raise TypeError("block_tables and context_lens must be int32")
    S, Hq, D = (int(x) for x in q.shape)
    P, Hkv, B, D2 = (int(x) for x in k_pool.shape)
    if tuple(out.shape) != (S, Hq, D) or tuple(v_pool.shape) != (P, Hkv, B, D2) or D2 != D:
        raise ValueError("shape mismatch between q/out/k_pool/v_pool")
    if block_tables.dim() != 2 or block_tables.shape[0] != S or tuple(context_lens.shape) != (S,):
        raise ValueError("block_tables must be [S][max_blocks] and context_lens [S]")
    need = decode_workspace_bytes(S, Hq, D, max_context_len, partition_size)
    if need and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    rc = lib.paged_attn_decode(
        _out_ptr(out, dev), _dev_ptr(q, "q", dev), _dev_ptr(k_pool, "k_pool", dev),
        _dev_ptr(v_pool, "v_pool", dev), _dev_ptr(block_tables, "block_tables", dev),
        _dev_ptr(context_lens, "context_lens", dev), S, Hq, Hkv, D, B,
        int(block_tables.shape[1]), P, int(max_context_len), float(scale), DTYPE_CODES[q.dtype],
        int(partition_size), _dev_ptr(workspace, "workspace", dev), ws_bytes,
        _dev_ptr(err, "err", dev), _stream_ptr(stream, dev))
    _check("paged_attn_decode", rc)
    return out


def paged_attn_decode_append(out: torch.Tensor, q: torch.Tensor, k_new: torch.Tensor,
                             v_new: torch.Tensor, k_pool: torch.Tensor, v_pool: torch.Tensor,
                             block_tables: torch.Tensor, context_lens: torch.Tensor,
                             scale: float, max_context_len: int,
                             partition_size: int = DEFAULT_PARTITION,
                             workspace: Optional[torch.Tensor] = None,
                             err: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """One decode step with the cache-append fused in: sequence s's newest token
    (``k_new[s]``, ``v_new[s]``, [S][Hkv][D]) is written into the pool slot of its
    token ``context_lens[s] - 1`` and attended over, in one pass (fp16/bf16)."""
    lib = load_library()
    _dev_ptr(q, "q")  # q decides the device every other tensor must be on
    dev = q.device
    if q.dtype not in DTYPE_CODES or any(t.dtype != q.dtype
                                         for t in (out, k_new, v_new, k_pool, v_pool)):
        raise TypeError("q, out, k_new, v_new and the pools must share one dtype")
    if block_tables.dtype != torch.int32 or context_lens.dtype != torch.int32:
        raise TypeError("block_tables and context_lens must be int32")
    S, Hq, D = (int(x) for x in q.shape)
    P, Hkv, B, D2 = (int(x) for x in k_pool.shape)
    if tuple(out.shape) != (S, Hq, D) or tuple(v_pool.shape) != (P, Hkv, B, D2) or D2 != D \
            or tuple(k_new.shape) != (S, Hkv, D) or tuple(v_new.shape) != (S, Hkv, D):
        raise ValueError("shape mismatch between q/out/k_new/v_new/pools")
    if block_tables.dim() != 2 or block_tables.shape[0] != S or tuple(context_lens.shape) != (S,):
        raise ValueError("block_tables must be [S][max_blocks] and context_lens [S]")
    need = decode_workspace_bytes(S, Hq, D, max_context_len, partition_size)
    if need and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    rc = lib.paged_attn_decode_append(
        _out_ptr(out, dev), _dev_ptr(q, "q", dev), _dev_ptr(k_new, "k_new", dev),
        _dev_ptr(v_new, "v_new", dev), _dev_ptr(k_pool, "k_pool", dev),
        _dev_ptr(v_pool, "v_pool", dev), _dev_ptr(block_tables, "block_tables", dev),
        _dev_ptr(context_lens, "context_lens", dev), S, Hq, Hkv, D, B,
        int(block_tables.shape[1]), P, int(max_context_len), float(scale), DTYPE_CODES[q.dtype],
        int(partition_size), _dev_ptr(workspace, "workspace", dev), ws_bytes,
        _dev_ptr(err, "err", dev), _stream_ptr(stream, dev))
    _check("paged_attn_decode_append", rc)
    return out


def kv_cache_append(k_pool: torch.Tensor, v_pool: torch.Tensor, k_new: torch.Tensor,
                    v_new: torch.Tensor, slot_mapping: torch.Tensor,
                    err: Optional[torch.Tensor] = None, stream=None) -> None:
    """Scatter ``k_new``/``v_new`` [T][Hkv][D] into pool slots ``slot_mapping`` (int64 [T])."""
    lib = load_library()
    dev = k_pool.device
    if k_pool.dtype not in DTYPE_CODES or any(t.dtype != k_pool.dtype
                                              for t in (v_pool, k_new, v_new)):
        raise TypeError("pools and new tokens must share one of float32/float16/bfloat16")
    if slot_mapping.dtype != torch.int64:
        raise TypeError("slot_mapping must be int64")
    P, Hkv, B, D = (int(x) for x in k_pool.shape)
    T = int(slot_mapping.shape[0])
    if tuple(k_new.shape) != (T, Hkv, D) or tuple(v_new.shape) != (T, Hkv, D) \
            or tuple(v_pool.shape) != (P, Hkv, B, D):
        raise ValueError("shape mismatch between pools, new tokens and slot_mapping")
    rc = lib.kv_cache_append(_dev_ptr(k_pool, "k_pool", dev), _dev_ptr(v_pool, "v_pool", dev),
                             _dev_ptr(k_new, "k_new", dev), _dev_ptr(v_new, "v_new", dev),
                             _dev_ptr(slot_mapping, "slot_mapping", dev), T, Hkv, D, B, P,
                             DTYPE_CODES[k_pool.dtype], _dev_ptr(err, "err", dev),
                             _stream_ptr(stream, dev))
    _check("kv_cache_append", rc)


def kv_block_copy(k_pool: torch.Tensor, v_pool: torch.Tensor, src_dst: torch.Tensor,
                  err: Optional[torch.Tensor] = None, stream=None) -> None:
    """Copy whole blocks ``src_dst[i] = (src, dst)`` (int32 [N][2]) in both pools."""
    lib = load_library()
    dev = k_pool.device
    if k_pool.dtype not in DTYPE_CODES or v_pool.dtype != k_pool.dtype:
        raise TypeError("pools must share one of float32/float16/bfloat16")
    if src_dst.dtype != torch.int32 or (src_dst.numel() and src_dst.dim() != 2):
        raise TypeError("src_dst must be int32 [N][2]")
    P, Hkv, B, D = (int(x) for x in k_pool.shape)
    N = int(src_dst.shape[0]) if src_dst.numel() else 0
    rc = lib.kv_block_copy(_dev_ptr(k_pool, "k_pool", dev), _dev_ptr(v_pool, "v_pool", dev),
                           _dev_ptr(src_dst, "src_dst", dev) if N else None, N, Hkv, D, B, P,
                           DTYPE_CODES[k_pool.dtype], _dev_ptr(err, "err", dev),
                           _stream_ptr(stream, dev))
    _check("kv_block_copy", rc)


def _dev_or_pinned_ptr(t: torch.Tensor, name: str, device):
    """A CUDA tensor on `device`, or a page-locked host tensor the device can
    address directly."""
    if isinstance(t, torch.Tensor) and t.device.type == "cpu":
        if not t.is_pinned():
            raise ValueError(f"{name} on the host must be pinned (page-locked) memory")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
        return ctypes.c_void_p(t.data_ptr())
    return _dev_ptr(t, name, device)


def kv_block_swap(dst_k: torch.Tensor, dst_v: torch.Tensor, src_k: torch.Tensor,
                  src_v: torch.Tensor, src_dst: torch.Tensor, err: Optional[torch.Tensor] = None,
                  stream=None, device=None) -> None:
    """Copy whole blocks ``src_dst[i] = (src, dst)`` (int32 [N][2]) from the
    source pools to the destination pools. Each pool, and ``src_dst``, may be
    on the GPU or in pinned host memory: swap-out is device -> host, swap-in
    host -> device."""
    lib = load_library()
    if device is None:
        cuda = [t for t in (dst_k, dst_v, src_k, src_v, src_dst) if t.device.type == "cuda"]
        device = cuda[0].device if cuda else torch.device("cuda", torch.cuda.current_device())
    dt = src_k.dtype
    if dt not in DTYPE_CODES or any(t.dtype != dt for t in (src_v, dst_k, dst_v)):
        raise TypeError("pools must share one of float32/float16/bfloat16")
    if src_dst.dtype != torch.int32:
        raise TypeError("src_dst must be int32")
    Ps, Hkv, B, D = (int(x) for x in src_k.shape)
    Pd = int(dst_k.shape[0])
    if tuple(src_v.shape) != (Ps, Hkv, B, D) or tuple(dst_k.shape[1:]) != (Hkv, B, D) \
            or tuple(dst_v.shape) != (Pd, Hkv, B, D):
        raise ValueError("pools must share the block shape [Hkv][B][D]")
    N = int(src_dst.shape[0]) if src_dst.numel() else 0
    if N and tuple(src_dst.shape) != (N, 2):
        raise ValueError("src_dst must be [N][2]")
    ptr = lambda t, n: _dev_or_pinned_ptr(t, n, device)
    rc = lib.kv_block_swap(ptr(dst_k, "dst_k"), ptr(dst_v, "dst_v"), ptr(src_k, "src_k"),
                           ptr(src_v, "src_v"), ptr(src_dst, "src_dst") if N else None, N, Hkv,
                           D, B, Ps, Pd, DTYPE_CODES[dt], _dev_ptr(err, "err", device),
                           _stream_ptr(stream, device))
    _check("kv_block_swap", rc)


def check_wait_timeout(err: torch.Tensor, limit_cycles: int = 2_000_000, stream=None) -> None:
    """Run the decode kernels' bounded wait on a barrier nothing completes; the
    wait gives up after ``limit_cycles`` and stores PKV_DEV_WAIT_TIMEOUT in err."""
    lib = load_library()
    rc = lib.pkv_check_wait_timeout(int(limit_cycles), _dev_ptr(err, "err", err.device),
                                    _stream_ptr(stream, err.device))
    _check("pkv_check_wait_timeout", rc)


def device_error_message(code: int) -> str:
    return DEV_ERRORS.get(int(code), f"code {int(code)}")
