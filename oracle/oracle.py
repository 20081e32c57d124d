"""ctypes wrapper around the fp64 CPU oracle (oracle.c).

TEST INFRASTRUCTURE ONLY: tests, the smoke check and the benchmark's CPU
baseline may import this module; the product path never does.  The oracle
shares no code with the CUDA library.  `build()` compiles oracle.c with gcc
into oracle/liboracle.so next to this file.
"""

from __future__ import annotations

import ctypes as C
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib: Optional[C.CDLL] = None

ERRORS = {0: "ok", 1: "invalid argument", 2: "slot, block id or length out of range", 3: "out of memory"}


class OracleError(RuntimeError):
    pass


def build(force: bool = False) -> str:
    """Compile oracle.c (plain C11, -O2, no fast-math) if the library is stale."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-std=c11", "-O2", "-fPIC", "-shared", "-pthread",
                               "-fno-fast-math", "-ffp-contract=off", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def load(path: str) -> C.CDLL:
    """Load an oracle build from `path` with its ctypes signatures set."""
    l = C.CDLL(path)
    p = C.c_void_p
    i32 = C.c_int32
    l.oracle_store_kvcache.argtypes = [p, p, C.c_int64, p, p, p, i32, i32, i32, i32, i32]
    l.oracle_store_kvcache.restype = C.c_int
    l.oracle_paged_attention.argtypes = [p, p, p, p, p, p, i32, p, i32, i32, i32, i32, i32, i32,
                                         C.c_double, i32]
    l.oracle_paged_attention.restype = C.c_int
    l.oracle_bf16_to_double.argtypes = [C.c_uint16]
    l.oracle_bf16_to_double.restype = C.c_double
    l.oracle_rope.argtypes = [p, p, C.c_int64, i32, i32, C.c_int64, p, C.c_double]
    l.oracle_rope.restype = C.c_int
    l.oracle_double_to_bf16.argtypes = [C.c_double]
    l.oracle_double_to_bf16.restype = C.c_uint16
    return l


def lib() -> C.CDLL:
    global _lib
    if _lib is None:
        _lib = load(build())
    return _lib


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


def _check(rc: int) -> None:
    if rc != 0:
        raise OracleError(f"oracle: {ERRORS.get(rc, rc)}")


def default_threads() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def store_kvcache(key: np.ndarray, value: np.ndarray, k_pool: np.ndarray, v_pool: np.ndarray,
                  slot_mapping: np.ndarray, _lib: Optional[C.CDLL] = None) -> None:
    """In-place store of new key/value rows into the [NB, BS, Hkv, D] uint16 pools."""
    key = np.ascontiguousarray(key, dtype=np.uint16)
    value = np.ascontiguousarray(value, dtype=np.uint16)
    slots = np.ascontiguousarray(slot_mapping, dtype=np.int32)
    assert k_pool.dtype == np.uint16 and k_pool.flags.c_contiguous and v_pool.flags.c_contiguous
    NB, BS, Hkv, D = k_pool.shape
    T = slots.shape[0]
    assert key.shape == (T, Hkv, D) and value.shape == (T, Hkv, D)
    _check((_lib or lib()).oracle_store_kvcache(_ptr(key), _ptr(value), Hkv * D, _ptr(k_pool), _ptr(v_pool),
                                      _ptr(slots), T, NB, BS, Hkv, D))


def paged_attention(q: np.ndarray, k_pool: np.ndarray, v_pool: np.ndarray, block_tables: np.ndarray,
                    context_lens: np.ndarray, cu_seqlens_q: np.ndarray, scale: float = 0.0,
                    threads: Optional[int] = None, _lib: Optional[C.CDLL] = None) -> np.ndarray:
    """fp64 attention of packed query rows [total_q, Hq, D] over the paged cache."""
    q = np.ascontiguousarray(q, dtype=np.uint16)
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    cl = np.ascontiguousarray(context_lens, dtype=np.int32)
    cu = np.ascontiguousarray(cu_seqlens_q, dtype=np.int32)
    assert k_pool.dtype == np.uint16 and k_pool.flags.c_contiguous and v_pool.flags.c_contiguous
    NB, BS, Hkv, D = k_pool.shape
    total_q, Hq, Dq = q.shape
    assert Dq == D
    B = cl.shape[0]
    assert cu.shape == (B + 1,) and int(cu[-1]) == total_q
    out = np.zeros((total_q, Hq, D), dtype=np.float64)
    mb = bt.shape[1] if bt.ndim == 2 else 0
    _check((_lib or lib()).oracle_paged_attention(_ptr(out), _ptr(q), _ptr(cu), _ptr(k_pool), _ptr(v_pool), _ptr(bt), mb,
                                        _ptr(cl), B, Hq, Hkv, D, NB, BS, float(scale),
                                        int(threads or default_threads())))
    return out


def decode_attention(q: np.ndarray, k_pool: np.ndarray, v_pool: np.ndarray, block_tables: np.ndarray,
                     context_lens: np.ndarray, scale: float = 0.0, threads: Optional[int] = None,
                     _lib: Optional[C.CDLL] = None) -> np.ndarray:
    """Decode: one query row per sequence, q [B, Hq, D]."""
    B = q.shape[0]
    cu = np.arange(B + 1, dtype=np.int32)
    return paged_attention(q, k_pool, v_pool, block_tables, context_lens, cu, scale, threads, _lib)


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to float64 (exact)."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def rope(x: np.ndarray, positions: np.ndarray, base: float, _lib: Optional[C.CDLL] = None) -> np.ndarray:
    """fp64 rotary embedding of bf16 rows x [T, H, D] at positions [T] (rotate-half pairing)."""
    x = np.ascontiguousarray(x, dtype=np.uint16)
    pos = np.ascontiguousarray(positions, dtype=np.int32)
    T, H, D = x.shape
    assert pos.shape == (T,)
    out = np.zeros((T, H, D), dtype=np.float64)
    _check((_lib or lib()).oracle_rope(_ptr(out), _ptr(x), T, H, D, H * D, _ptr(pos), float(base)))
    return out


def to_bf16(v: np.ndarray, _lib: Optional[C.CDLL] = None) -> np.ndarray:
    """Round fp64 values to bf16 bit patterns, nearest with ties to even."""
    f = (_lib or lib()).oracle_double_to_bf16
    flat = np.asarray(v, dtype=np.float64).ravel()
    return np.fromiter((f(float(a)) for a in flat), dtype=np.uint16, count=flat.size).reshape(np.shape(v))


def rope_store_kvcache(q: Optional[np.ndarray], key: np.ndarray, value: np.ndarray, positions: np.ndarray,
                       k_pool: np.ndarray, v_pool: np.ndarray, slot_mapping: np.ndarray, base: float,
                       _lib: Optional[C.CDLL] = None):
    """RoPE on q and key, then the store of the rotated key and the value.

    The tensors are bf16, so the rotated rows are the bf16 roundings of the fp64
    rotations.  Returns (q rotated [T, Hq, D] bf16 bits or None, fp64 rotated q,
    fp64 rotated key); the pools are updated in place.
    """
    kr = rope(key, positions, base, _lib)
    store_kvcache(to_bf16(kr, _lib), value, k_pool, v_pool, slot_mapping, _lib=_lib)
    if q is None:
        return None, None, kr
    qr = rope(q, positions, base, _lib)
    return to_bf16(qr, _lib), qr, kr
