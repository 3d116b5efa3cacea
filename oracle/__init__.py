"""CPU oracle for paged decode attention (test infrastructure only).

This is the slow, plain, fp64 reference for the hot path. It lives in
``pkv_oracle.c`` and is reached through ctypes. Only the tests, the smoke check
and the benchmark's CPU baseline use it. The library under
``paged_kv_cache_387_b200`` neither imports it nor shares code with it.

Each function names the passage it follows in the C source. Inputs are CPU
torch tensors, or numpy arrays, in the pool layout
``[num_blocks][num_kv_heads][block_size][head_dim]``. Outputs are numpy float64.
"""

from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pkv_oracle.c")
_LIB_DIR = os.path.join(_HERE, "_build")
_LIB = os.path.join(_LIB_DIR, "liboracle.so")

F32, F16, BF16 = 0, 1, 2
_ERRORS = {-1: "bad argument", -2: "block id or slot out of range", -3: "out of memory"}

_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, OpenMP, no fast-math)."""
    os.makedirs(_LIB_DIR, exist_ok=True)
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        I = ctypes.c_int
        D = ctypes.c_double
        lib.oracle_paged_decode.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, I, D, I]
        lib.oracle_paged_decode_blockwise.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, I, D, I]
        lib.oracle_paged_decode_partitioned.argtypes = [P, P, P, I, P, P, P, P, P,
                                                        I, I, I, I, I, I, I, D, I, I]
        lib.oracle_cache_append.argtypes = [P, P, P, P, P, I, I, I, I, I, I]
        lib.oracle_block_copy.argtypes = [P, P, P, I, I, I, I, I, I]
        lib.oracle_block_swap.argtypes = [P, P, P, P, P, I, I, I, I, I, I, I]
        lib.oracle_half_to_double.argtypes = [ctypes.c_uint16]
        lib.oracle_half_to_double.restype = D
        lib.oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
        lib.oracle_bf16_to_double.restype = D
        lib.oracle_num_threads.restype = I
        for f in ("oracle_paged_decode", "oracle_paged_decode_blockwise",
                  "oracle_paged_decode_partitioned", "oracle_cache_append",
                  "oracle_block_copy", "oracle_block_swap"):
            getattr(lib, f).restype = I
        _lib = lib
    return _lib


def _dtype_code(t) -> Tuple[int, int]:
    name = str(t.dtype)
    if name in ("torch.float32", "float32"):
        return F32, 4
    if name in ("torch.float16", "float16"):
        return F16, 2
    if name in ("torch.bfloat16",):
        return BF16, 2
    raise TypeError(f"unsupported dtype {t.dtype}")


def _ptr(t):
    """Address of a contiguous CPU torch tensor or numpy array."""
    if hasattr(t, "data_ptr"):
        if t.device.type != "cpu" or not t.is_contiguous():
            raise ValueError("oracle inputs must be contiguous CPU tensors")
        return ctypes.c_void_p(t.data_ptr())
    if not t.flags["C_CONTIGUOUS"]:
        raise ValueError("oracle inputs must be C-contiguous")
    return ctypes.c_void_p(t.ctypes.data)


def _check(rc: int, what: str):
    if rc != 0:
        raise RuntimeError(f"oracle {what}: {_ERRORS.get(rc, rc)}")


def _shapes(q, k_pool, block_tables):
    S, Hq, D = (int(x) for x in q.shape)
    P, Hkv, B, D2 = (int(x) for x in k_pool.shape)
    if D2 != D:
        raise ValueError("head_dim mismatch between q and pools")
    return S, Hq, D, P, Hkv, B, int(block_tables.shape[1]) if block_tables.ndim == 2 else 0


def half_to_double(bits: int) -> float:
    return _load().oracle_half_to_double(bits)


def bf16_to_double(bits: int) -> float:
    return _load().oracle_bf16_to_double(bits)


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def paged_decode(q, k_pool, v_pool, block_tables, context_lens, scale: float,
                 return_lse: bool = False):
    """Two-pass attention per (sequence, query head), fp64. Returns [S][Hq][D]."""
    lib = _load()
    S, Hq, D, P, Hkv, B, MB = _shapes(q, k_pool, block_tables)
    code, _ = _dtype_code(q)
    out = np.zeros((S, Hq, D), np.float64)
    lse = np.zeros((S, Hq), np.float64) if return_lse else None
    rc = lib.oracle_paged_decode(_ptr(out), _ptr(lse) if lse is not None else None,
                                 _ptr(q), _ptr(k_pool), _ptr(v_pool), _ptr(block_tables),
                                 _ptr(context_lens), S, Hq, Hkv, D, B, MB, P, float(scale), code)
    _check(rc, "paged_decode")
    return (out, lse) if return_lse else out


def paged_decode_blockwise(q, k_pool, v_pool, block_tables, context_lens, scale: float):
    """Block-by-block online-softmax walk over the block table, fp64."""
    lib = _load()
    S, Hq, D, P, Hkv, B, MB = _shapes(q, k_pool, block_tables)
    code, _ = _dtype_code(q)
    out = np.zeros((S, Hq, D), np.float64)
    rc = lib.oracle_paged_decode_blockwise(_ptr(out), _ptr(q), _ptr(k_pool), _ptr(v_pool),
                                           _ptr(block_tables), _ptr(context_lens),
                                           S, Hq, Hkv, D, B, MB, P, float(scale), code)
    _check(rc, "paged_decode_blockwise")
    return out


def paged_decode_partitioned(q, k_pool, v_pool, block_tables, context_lens, scale: float,
                             partition_size: int, max_parts: Optional[int] = None):
    """Split-context attention + log-sum-exp combine, fp64.

    Returns ``(out [S][Hq][D], part_o [S][Hq][max_parts][D], part_lse [S][Hq][max_parts])``.
    """
    lib = _load()
    S, Hq, D, P, Hkv, B, MB = _shapes(q, k_pool, block_tables)
    code, _ = _dtype_code(q)
    lens = np.asarray(context_lens)
    if max_parts is None:
        max_parts = max(1, int(-(-int(lens.max()) // partition_size))) if S else 1
    out = np.zeros((S, Hq, D), np.float64)
    po = np.zeros((S, Hq, max_parts, D), np.float64)
    pl = np.zeros((S, Hq, max_parts), np.float64)
    rc = lib.oracle_paged_decode_partitioned(_ptr(out), _ptr(po), _ptr(pl), int(max_parts),
                                             _ptr(q), _ptr(k_pool), _ptr(v_pool),
                                             _ptr(block_tables), _ptr(context_lens),
                                             S, Hq, Hkv, D, B, MB, P, float(scale), code,
                                             int(partition_size))
    _check(rc, "paged_decode_partitioned")
    return out, po, pl


def cache_append(k_pool, v_pool, k_new, v_new, slot_mapping) -> None:
    """In-place CPU scatter of new tokens' K/V into their pool slots."""
    lib = _load()
    P, Hkv, B, D = (int(x) for x in k_pool.shape)
    T = int(slot_mapping.shape[0])
    _, es = _dtype_code(k_pool)
    rc = lib.oracle_cache_append(_ptr(k_pool), _ptr(v_pool), _ptr(k_new), _ptr(v_new),
                                 _ptr(slot_mapping), T, Hkv, D, B, P, es)
    _check(rc, "cache_append")


def block_swap(dst_k, dst_v, src_k, src_v, pairs) -> None:
    """CPU whole-block copies from block src of the source pools into block
    dst of the destination pools (K and V)."""
    lib = _load()
    Ps, Hkv, B, D = (int(x) for x in src_k.shape)
    Pd = int(dst_k.shape[0])
    _, es = _dtype_code(src_k)
    n = int(pairs.shape[0]) if pairs.ndim == 2 else 0
    rc = lib.oracle_block_swap(_ptr(dst_k), _ptr(dst_v), _ptr(src_k), _ptr(src_v), _ptr(pairs), n,
                               Hkv, D, B, Ps, Pd, es)
    _check(rc, "block_swap")


def block_copy(k_pool, v_pool, pairs) -> None:
    """In-place CPU whole-block copies src -> dst for both pools."""
    lib = _load()
    P, Hkv, B, D = (int(x) for x in k_pool.shape)
    _, es = _dtype_code(k_pool)
    n = int(pairs.shape[0]) if pairs.ndim == 2 else 0
    rc = lib.oracle_block_copy(_ptr(k_pool), _ptr(v_pool), _ptr(pairs), n, Hkv, D, B, P, es)
    _check(rc, "block_copy")
