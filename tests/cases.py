"""Small seeded cases shared by the oracle pins and the GPU parity tests."""

from __future__ import annotations

from typing import Optional, Tuple

import numpy as np

from paged_kv_cache_bf16_b200 import workloads as W


def tiny_spec(name: str = "tiny", seed: int = 101, **kw) -> W.Spec:
    base = dict(name=name, seed=seed, num_seqs=4, num_q_heads=4, num_kv_heads=2, head_dim=8, block_size=4,
                num_blocks=64, ctx_lo=1, ctx_hi=14)
    base.update(kw)
    return W.Spec(**base)


def oracle_post_store(wl: W.Workload, step: int = 0, lib=None) -> Tuple[np.ndarray, np.ndarray]:
    """Host pools after the oracle applied the stores of steps 0..step."""
    from oracle import oracle as O

    kp, vp = wl.host_pool()
    for s in range(step + 1):
        k, v = wl.new_kv(s)
        O.store_kvcache(k, v, kp, vp, wl.slot_mapping(s), _lib=lib)
    return kp, vp


def oracle_attention(wl: W.Workload, kp: np.ndarray, vp: np.ndarray, step: int = 0, lib=None,
                     scale: float = 0.0, threads: Optional[int] = None) -> np.ndarray:
    from oracle import oracle as O

    return O.paged_attention(wl.q(step), kp, vp, wl.block_tables(step), wl.context_lens(step),
                             wl.cu_seqlens_q(), scale=scale, threads=threads, _lib=lib)


def oracle_compact(wl: W.Workload, step: int = 0, seqs=None, lib=None, threads: Optional[int] = None,
                   scale: float = 0.0):
    """Oracle outputs for sequences `seqs` (default: all) at `step`.

    The oracle gets a pool holding only the blocks those sequences reference,
    relabelled 0..n-1 in order of first use (relabelling is a pinned invariant),
    the cached prefixes, and every store of steps 0..step applied by the
    oracle's own store.  Returns (fp64 out [rows, Hq, D], packed row indices).
    """
    from oracle import oracle as O

    seqs = list(range(wl.B)) if seqs is None else [int(b) for b in seqs]
    L = wl.context_lens(step)
    bt = wl.block_tables(step)
    remap = {}
    bt_c = np.full((len(seqs), wl.max_blocks_per_seq), -1, dtype=np.int32)
    for r, b in enumerate(seqs):
        for i in range(-(-int(L[b]) // wl.BS)):
            p = int(bt[b, i])
            if p not in remap:
                remap[p] = len(remap)
            bt_c[r, i] = remap[p]
    n = max(1, len(remap))
    shape = (n, wl.BS, wl.Hkv, wl.D)
    kp = np.full(shape, W.BF16_NAN, dtype=np.uint16)
    vp = np.full(shape, W.BF16_NAN, dtype=np.uint16)
    for p, nv in wl.prior_fill():
        if p in remap:
            k, v = wl.block_contents(p, nv)
            kp[remap[p], :nv] = k
            vp[remap[p], :nv] = v
    chosen = np.zeros(wl.B, dtype=bool)
    chosen[seqs] = True
    for s in range(step + 1):
        seq_of_tok, _ = wl.token_positions(s)
        keep = chosen[seq_of_tok]
        slots = wl.slot_mapping(s)[keep]
        k, v = wl.new_kv(s)
        cslots = np.array([remap[int(x) // wl.BS] * wl.BS + int(x) % wl.BS for x in slots], dtype=np.int32)
        O.store_kvcache(k[keep], v[keep], kp, vp, cslots, _lib=lib)
    cu = wl.cu_seqlens_q()
    rows = np.concatenate([np.arange(cu[b], cu[b + 1]) for b in seqs]) if seqs else np.zeros(0, np.int64)
    qsub = wl.q(step)[rows]
    cu_c = np.zeros(len(seqs) + 1, dtype=np.int32)
    cu_c[1:] = np.cumsum(wl.query_lens[seqs])
    out = O.paged_attention(qsub, kp, vp, bt_c, L[seqs], cu_c, scale=scale, threads=threads, _lib=lib)
    return out, rows
