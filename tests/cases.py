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


def compact_seq_pool(wl: W.Workload, b: int, step: int, kp_full=None, vp_full=None):
    """The blocks of sequence b (after stores up to `step`) relabelled 0..n-1.

    Physical relabelling leaves attention unchanged (a pinned oracle property),
    so a compact pool stands in for a 4,096- or 57,344-block pool when the
    oracle checks sampled sequences of a full-size workload.
    Returns (k_pool, v_pool, block_table_row, context_len).
    """
    L = int(wl.context_lens(step)[b])
    nblk = -(-L // wl.BS)
    blocks = [int(p) for p in wl.seq_blocks[b][:nblk]]
    shape = (nblk, wl.BS, wl.Hkv, wl.D)
    kp = np.full(shape, W.BF16_NAN, dtype=np.uint16)
    vp = np.full(shape, W.BF16_NAN, dtype=np.uint16)
    if kp_full is not None:
        kp[:] = kp_full[blocks]
        vp[:] = vp_full[blocks]
        return kp, vp, np.arange(nblk, dtype=np.int32), L
    # cached prefix from the generator, then every new token stored up to `step`
    pl = wl.prior_len(b)
    for i, p in enumerate(blocks):
        n = max(0, min(wl.BS, pl - i * wl.BS))
        if n:
            k, v = wl.block_contents(p, n)
            kp[i, :n] = k
            vp[i, :n] = v
    hd = wl.Hkv * wl.D
    j0 = pl
    n_new = L - pl
    if n_new > 0:
        k = W.normal_bf16(W.stream_key(wl.spec.seed, W.TAG_NEW_K, b), j0 * hd, n_new * hd, wl.spec.sigma)
        v = W.normal_bf16(W.stream_key(wl.spec.seed, W.TAG_NEW_V, b), j0 * hd, n_new * hd, wl.spec.sigma)
        k = k.reshape(n_new, wl.Hkv, wl.D)
        v = v.reshape(n_new, wl.Hkv, wl.D)
        for t in range(n_new):
            j = j0 + t
            kp[j // wl.BS, j % wl.BS] = k[t]
            vp[j // wl.BS, j % wl.BS] = v[t]
    return kp, vp, np.arange(nblk, dtype=np.int32), L
