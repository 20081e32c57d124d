"""A second, separately written fp64 reference in pure Python, for tiny inputs.

It shares nothing with oracle/oracle.c: it walks each sequence's block table
block by block to rebuild the contiguous key/value sequence, loops over KV heads
and the query heads each one serves, and normalises through a log-sum-exp
rather than a division.  Used only to pin the oracle.
"""

from __future__ import annotations

import math
import struct
from typing import List


def bf16(bits: int) -> float:
    return struct.unpack("<f", struct.pack("<I", (int(bits) & 0xFFFF) << 16))[0]


def attention(q, k_pool, v_pool, block_tables, context_lens, cu_seqlens_q, scale=None) -> List:
    """q [total_q][Hq][D] bf16 bits, pools [NB][BS][Hkv][D] bits -> nested fp64 lists."""
    NB, BS, Hkv, D = k_pool.shape
    Hq = q.shape[1]
    g = Hq // Hkv
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    out = [[[0.0] * D for _ in range(Hq)] for _ in range(q.shape[0])]
    for b in range(len(context_lens)):
        L = int(context_lens[b])
        n = int(cu_seqlens_q[b + 1]) - int(cu_seqlens_q[b])
        keys, vals = [], []
        logical = 0
        while len(keys) < L:
            phys = int(block_tables[b][logical])
            for off in range(BS):
                if len(keys) == L:
                    break
                keys.append([[bf16(k_pool[phys, off, h, d]) for d in range(D)] for h in range(Hkv)])
                vals.append([[bf16(v_pool[phys, off, h, d]) for d in range(D)] for h in range(Hkv)])
            logical += 1
        for hk in range(Hkv):
            for hq in range(hk * g, (hk + 1) * g):
                for i in range(n):
                    r = int(cu_seqlens_q[b]) + i
                    qv = [bf16(q[r, hq, d]) for d in range(D)]
                    last = L - n + i
                    s = [scale * math.fsum(qv[d] * keys[j][hk][d] for d in range(D)) for j in range(last + 1)]
                    m = max(s)
                    lse = m + math.log(math.fsum(math.exp(x - m) for x in s))
                    w = [math.exp(x - lse) for x in s]
                    out[r][hq] = [math.fsum(w[j] * vals[j][hk][d] for j in range(last + 1)) for d in range(D)]
    return out
