"""Thin Python binding of libnpv (include/npv.h).

Argument marshalling only: every step of the attention path runs in the CUDA
kernels of libnpv.so.  Tensors are torch CUDA tensors (PyTorch supplies device
memory and streams); calls run on torch's current stream.  There is no CPU
fallback: if libnpv.so is missing, loading it raises.
"""

from __future__ import annotations

import ctypes as C
import math
import os
import re
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libnpv.so")
HEADER = os.path.join(os.path.dirname(_HERE), "include", "npv.h")

NPV_OK = 0
STATUS_NAMES = {0: "NPV_OK", 1: "NPV_ERR_INVALID_ARG", 2: "NPV_ERR_UNSUPPORTED", 3: "NPV_ERR_WORKSPACE",
                4: "NPV_ERR_CUDA", 5: "NPV_ERR_DEVICE_BOUNDS"}
DEVERR_BITS = {0x1: "SLOT", 0x2: "BLOCK_ID", 0x4: "CONTEXT_LEN", 0x8: "QUERY_LENS", 0x10: "TIMEOUT"}

_lib: Optional[C.CDLL] = None


class NpvError(RuntimeError):
    def __init__(self, status: int, what: str, bits: int = 0):
        self.status = status
        self.bits = bits
        msg = f"{what}: {STATUS_NAMES.get(status, status)} ({lib().npv_status_string(status).decode()})"
        if bits:
            msg += " bits=" + "|".join(n for b, n in DEVERR_BITS.items() if bits & b)
        super().__init__(msg)


def exported_symbols() -> list:
    """Names of the functions include/npv.h declares."""
    text = open(HEADER).read()
    return re.findall(r"NPV_API\s+[\w\s\*]+?\b(npv_\w+)\s*\(", text)


def lib() -> C.CDLL:
    """The loaded libnpv.so with ctypes signatures (raises if it is not built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing; build it with `python -m paged_kv_cache_bf16_b200.build`")
    l = C.CDLL(LIB_PATH)
    p, i32, i64, sz = C.c_void_p, C.c_int32, C.c_int64, C.c_size_t
    l.npv_status_string.argtypes = [C.c_int]
    l.npv_status_string.restype = C.c_char_p
    l.npv_version.argtypes = []
    l.npv_version.restype = C.c_int
    l.npv_store_kvcache.argtypes = [p, p, i64, i64, p, p, p, i32, i32, i32, i32, i32, p]
    l.npv_store_kvcache.restype = C.c_int
    l.npv_rope_store_kvcache.argtypes = [p, i64, i32, p, p, i64, i64, p, p, p, p, i32, i32, i32, i32, i32,
                                         C.c_double, p]
    l.npv_rope_store_kvcache.restype = C.c_int
    l.npv_paged_decode_workspace_size.argtypes = [i32, i32, i32, i32]
    l.npv_paged_decode_workspace_size.restype = sz
    l.npv_paged_decode_attention.argtypes = [p, p, i64, p, p, p, i32, p, i32, i32, i32, i32, i32, i32, C.c_float,
                                             p, sz, p]
    l.npv_paged_decode_attention.restype = C.c_int
    l.npv_store_kvcache_and_decode_attention.argtypes = [p, p, i64, p, p, i64, i64, p, p, p, p, i32, p, i32, i32,
                                                         i32, i32, i32, i32, C.c_float, p, sz, p]
    l.npv_store_kvcache_and_decode_attention.restype = C.c_int
    l.npv_paged_prefill_workspace_size.argtypes = [i32, i32, i32, i32, i32]
    l.npv_paged_prefill_workspace_size.restype = sz
    l.npv_paged_prefill_attention.argtypes = [p, p, p, i32, i32, p, p, p, i32, p, i32, i32, i32, i32, i32, i32,
                                              C.c_float, p, sz, p]
    l.npv_paged_prefill_attention.restype = C.c_int
    l.npv_check_device_errors.argtypes = [p, C.POINTER(C.c_uint32)]
    l.npv_check_device_errors.restype = C.c_int
    l.npv_debug_inject_decode_timeout.argtypes = [C.c_int]
    l.npv_debug_inject_decode_timeout.restype = C.c_int
    _lib = l
    return l


def _check(status: int, what: str) -> None:
    if status != NPV_OK:
        raise NpvError(status, what)


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _on_one_gpu(what: str, bf16=(), other=()) -> None:
    """Every tensor a call hands to the kernels must live on one CUDA device (a host
    pointer would be dereferenced by the GPU); the activation and cache tensors must
    be bf16.  Raises before anything is launched."""
    dev = None
    for name, t in list(bf16) + list(other):
        if t is None:
            continue
        if not isinstance(t, torch.Tensor) or not t.is_cuda:
            raise ValueError(f"{what}: {name} must be a CUDA tensor")
        if dev is None:
            dev = t.device
        elif t.device != dev:
            raise ValueError(f"{what}: {name} is on {t.device}, the other tensors on {dev}")
    for name, t in bf16:
        if t is not None and t.dtype != torch.bfloat16:
            raise TypeError(f"{what}: {name} must be torch.bfloat16, got {t.dtype}")


def _cache_shape(k_cache: torch.Tensor):
    assert k_cache.dim() == 4 and k_cache.is_contiguous(), "cache must be [num_blocks, block_size, Hkv, D]"
    return k_cache.shape


def store_kvcache(key: torch.Tensor, value: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                  slot_mapping: torch.Tensor, stream=None) -> None:
    """Scatter key/value [T, Hkv, D] bf16 into the caches at slot_mapping [T] int32."""
    _on_one_gpu("store_kvcache", bf16=[("key", key), ("value", value), ("k_cache", k_cache), ("v_cache", v_cache)],
                other=[("slot_mapping", slot_mapping)])
    NB, BS, Hkv, D = _cache_shape(k_cache)
    T = slot_mapping.shape[0]
    assert slot_mapping.dtype == torch.int32
    assert key.shape[0] == T and value.shape[0] == T
    assert key.stride(-1) == 1 and key.stride(-2) == D and value.stride(-1) == 1 and value.stride(-2) == D
    _check(lib().npv_store_kvcache(_ptr(key), _ptr(value), key.stride(0) if T else 0, value.stride(0) if T else 0,
                                   _ptr(k_cache), _ptr(v_cache), _ptr(slot_mapping), T, NB, BS, Hkv, D,
                                   _stream(stream)), "npv_store_kvcache")


def rope_store_kvcache(q: Optional[torch.Tensor], key: torch.Tensor, value: torch.Tensor, positions: torch.Tensor,
                       k_cache: torch.Tensor, v_cache: torch.Tensor, slot_mapping: torch.Tensor, rope_base: float,
                       stream=None) -> None:
    """RoPE on q (in place, [T, Hq, D]; None for none) and key [T, Hkv, D] at positions [T] int32,
    then the store of the rotated key and of value [T, Hkv, D] at slot_mapping [T] int32."""
    _on_one_gpu("rope_store_kvcache",
                bf16=[("q", q), ("key", key), ("value", value), ("k_cache", k_cache), ("v_cache", v_cache)],
                other=[("positions", positions), ("slot_mapping", slot_mapping)])
    NB, BS, Hkv, D = _cache_shape(k_cache)
    T = slot_mapping.shape[0]
    assert slot_mapping.dtype == torch.int32 and positions.dtype == torch.int32 and positions.shape == (T,)
    assert key.shape[0] == T and value.shape[0] == T
    assert key.stride(-1) == 1 and key.stride(-2) == D and value.stride(-1) == 1 and value.stride(-2) == D
    Hq = 0 if q is None else q.shape[1]
    if q is not None:
        assert q.shape[0] == T and q.shape[2] == D and q.stride(-1) == 1 and q.stride(-2) == D
    _check(lib().npv_rope_store_kvcache(_ptr(q) if q is not None else None, q.stride(0) if (q is not None and T) else 0,
                                        Hq, _ptr(key), _ptr(value), key.stride(0) if T else 0,
                                        value.stride(0) if T else 0, _ptr(positions), _ptr(k_cache), _ptr(v_cache),
                                        _ptr(slot_mapping), T, NB, BS, Hkv, D, float(rope_base), _stream(stream)),
           "npv_rope_store_kvcache")


def decode_workspace_size(num_seqs: int, num_q_heads: int, num_kv_heads: int, head_dim: int) -> int:
    return int(lib().npv_paged_decode_workspace_size(num_seqs, num_q_heads, num_kv_heads, head_dim))


def prefill_workspace_size(num_seqs: int, total_q: int, num_q_heads: int, num_kv_heads: int, head_dim: int) -> int:
    return int(lib().npv_paged_prefill_workspace_size(num_seqs, total_q, num_q_heads, num_kv_heads, head_dim))


def alloc_workspace(nbytes: int, device) -> torch.Tensor:
    # torch's caching allocator returns 512-byte aligned blocks
    return torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)


def paged_decode_attention(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                           block_tables: torch.Tensor, context_lens: torch.Tensor, scale: Optional[float] = None,
                           out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                           stream=None) -> torch.Tensor:
    """Decode attention: q [B, Hq, D] bf16 -> out [B, Hq, D] bf16."""
    _on_one_gpu("paged_decode_attention",
                bf16=[("q", q), ("k_cache", k_cache), ("v_cache", v_cache), ("out", out)],
                other=[("block_tables", block_tables), ("context_lens", context_lens), ("workspace", workspace)])
    NB, BS, Hkv, D = _cache_shape(k_cache)
    B, Hq, Dq = q.shape
    assert Dq == D and q.stride(2) == 1 and q.stride(1) == D
    assert block_tables.dtype == torch.int32 and context_lens.dtype == torch.int32 and block_tables.is_contiguous()
    if out is None:
        out = torch.empty((B, Hq, D), dtype=q.dtype, device=q.device)
    if workspace is None:
        workspace = alloc_workspace(decode_workspace_size(B, Hq, Hkv, D), q.device)
    _check(lib().npv_paged_decode_attention(_ptr(out), _ptr(q), q.stride(0), _ptr(k_cache), _ptr(v_cache),
                                            _ptr(block_tables), block_tables.shape[1], _ptr(context_lens), B, Hq,
                                            Hkv, D, NB, BS, float(scale or 0.0), _ptr(workspace),
                                            workspace.numel(), _stream(stream)), "npv_paged_decode_attention")
    return out


def store_kvcache_and_decode_attention(q: torch.Tensor, key: torch.Tensor, value: torch.Tensor,
                                       k_cache: torch.Tensor, v_cache: torch.Tensor, slot_mapping: torch.Tensor,
                                       block_tables: torch.Tensor, context_lens: torch.Tensor,
                                       scale: Optional[float] = None, out: Optional[torch.Tensor] = None,
                                       workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """One decode step in one launch set: store key/value [B, Hkv, D] at slot_mapping [B], then
    decode attention for q [B, Hq, D] -> out [B, Hq, D]."""
    _on_one_gpu("store_kvcache_and_decode_attention",
                bf16=[("q", q), ("key", key), ("value", value), ("k_cache", k_cache), ("v_cache", v_cache),
                      ("out", out)],
                other=[("slot_mapping", slot_mapping), ("block_tables", block_tables), ("context_lens", context_lens),
                       ("workspace", workspace)])
    NB, BS, Hkv, D = _cache_shape(k_cache)
    B, Hq, Dq = q.shape
    assert Dq == D and q.stride(2) == 1 and q.stride(1) == D
    assert key.shape == (B, Hkv, D) and value.shape == (B, Hkv, D) and slot_mapping.shape == (B,)
    assert key.stride(-1) == 1 and key.stride(-2) == D and value.stride(-1) == 1 and value.stride(-2) == D
    assert slot_mapping.dtype == torch.int32 and block_tables.dtype == torch.int32 and block_tables.is_contiguous()
    if out is None:
        out = torch.empty((B, Hq, D), dtype=q.dtype, device=q.device)
    if workspace is None:
        workspace = alloc_workspace(decode_workspace_size(B, Hq, Hkv, D), q.device)
    _check(lib().npv_store_kvcache_and_decode_attention(
        _ptr(out), _ptr(q), q.stride(0), _ptr(key), _ptr(value), key.stride(0), value.stride(0), _ptr(slot_mapping),
        _ptr(k_cache), _ptr(v_cache), _ptr(block_tables), block_tables.shape[1], _ptr(context_lens), B, Hq, Hkv, D,
        NB, BS, float(scale or 0.0), _ptr(workspace), workspace.numel(), _stream(stream)),
        "npv_store_kvcache_and_decode_attention")
    return out


def paged_prefill_attention(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                            cu_seqlens_q: torch.Tensor, max_seqlen_q: int, block_tables: torch.Tensor,
                            context_lens: torch.Tensor, scale: Optional[float] = None,
                            out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                            stream=None) -> torch.Tensor:
    """Varlen causal attention: q [total_q, Hq, D] packed by cu_seqlens_q -> out [total_q, Hq, D]."""
    _on_one_gpu("paged_prefill_attention",
                bf16=[("q", q), ("k_cache", k_cache), ("v_cache", v_cache), ("out", out)],
                other=[("cu_seqlens_q", cu_seqlens_q), ("block_tables", block_tables), ("context_lens", context_lens),
                       ("workspace", workspace)])
    NB, BS, Hkv, D = _cache_shape(k_cache)
    total_q, Hq, Dq = q.shape
    B = context_lens.shape[0]
    assert Dq == D and q.is_contiguous()
    assert cu_seqlens_q.dtype == torch.int32 and cu_seqlens_q.shape[0] == B + 1
    if out is None:
        out = torch.empty((total_q, Hq, D), dtype=q.dtype, device=q.device)
    if workspace is None:
        workspace = alloc_workspace(prefill_workspace_size(B, total_q, Hq, Hkv, D), q.device)
    _check(lib().npv_paged_prefill_attention(_ptr(out), _ptr(q), _ptr(cu_seqlens_q), int(max_seqlen_q), total_q,
                                             _ptr(k_cache), _ptr(v_cache), _ptr(block_tables),
                                             block_tables.shape[1], _ptr(context_lens), B, Hq, Hkv, D, NB, BS,
                                             float(scale or 0.0), _ptr(workspace), workspace.numel(),
                                             _stream(stream)), "npv_paged_prefill_attention")
    return out


def check_device_errors(stream=None) -> int:
    """Synchronise, then read and clear the device error word; raises NpvError if any bit was set."""
    bits = C.c_uint32(0)
    st = lib().npv_check_device_errors(_stream(stream), C.byref(bits))
    if st != NPV_OK:
        raise NpvError(st, "npv_check_device_errors", bits.value)
    return bits.value


def inject_decode_timeout(enable: bool) -> None:
    """Failure-detection test hook: make the decode kernel's bounded pipeline wait give up
    (see npv_debug_inject_decode_timeout in include/npv.h)."""
    _check(lib().npv_debug_inject_decode_timeout(1 if enable else 0), "npv_debug_inject_decode_timeout")


def default_scale(head_dim: int) -> float:
    return 1.0 / math.sqrt(head_dim)
