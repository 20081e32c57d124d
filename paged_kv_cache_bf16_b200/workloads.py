"""Seeded synthetic inputs for paged KV-cache attention.

This module only *draws* inputs.  It produces the integer metadata an engine's
runner would build (context lengths, query lengths, block tables drawn from a
shuffled free list, slot mappings, cu_seqlens_q) and the bf16 contents of
queries, new keys/values and cached keys/values.  It holds none of the
attention arithmetic: the CUDA path and the CPU oracle each do their own.

Random numbers come from SplitMix64 (Steele, Lea and Flood, "Fast splittable
pseudorandom number generators", OOPSLA 2014; the 64-bit finaliser published
by Vigna), used in counter form so that any element of any tensor can be
regenerated on its own.  Normal draws use the Box-Muller transform (one output
per pair of uniforms) and are rounded to bf16 with round-to-nearest-even.

The five named workloads follow the shapes of the pages' engine: Qwen3-0.6B
attention heads with 256-token blocks and 256 concurrent sequences
("Nano-vLLM Architecture and Performance", Key Features 2 and Performance),
LLaMA-8B-style 32:8 GQA heads ("nano-vllm" README, X-Ray Mode), prefix-shared
blocks (same page, Features: Prefix Caching) and 512-token prefill chunks (same
page, CLI options: --max-prefill-tokens).
"""

from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field
from typing import Dict, List, Optional, Tuple

import numpy as np

MASK64 = (1 << 64) - 1
GOLDEN = 0x9E3779B97F4A7C15
_MUL1 = 0xBF58476D1CE4E5B9
_MUL2 = 0x94D049BB133111EB

# bf16 quiet NaN used to poison every cache slot that holds no token.
BF16_NAN = np.uint16(0x7FC0)

# stream tags
TAG_META = 1
TAG_POOL_K = 2
TAG_POOL_V = 3
TAG_NEW_K = 4
TAG_NEW_V = 5
TAG_Q = 6


def mix64(z: int) -> int:
    """SplitMix64 output finaliser on a Python int."""
    z &= MASK64
    z = ((z ^ (z >> 30)) * _MUL1) & MASK64
    z = ((z ^ (z >> 27)) * _MUL2) & MASK64
    return z ^ (z >> 31)


def _mix64_np(z: np.ndarray) -> np.ndarray:
    with np.errstate(over="ignore"):
        z = (z ^ (z >> np.uint64(30))) * np.uint64(_MUL1)
        z = (z ^ (z >> np.uint64(27))) * np.uint64(_MUL2)
        return z ^ (z >> np.uint64(31))


def stream_key(*parts: int) -> int:
    """Fold integer parts into one 64-bit stream key."""
    k = 0x5EED
    for p in parts:
        k = mix64((k ^ (int(p) & MASK64)) + GOLDEN)
    return k


class SplitMix64:
    """Sequential SplitMix64 for small integer draws (lengths, permutations)."""

    def __init__(self, seed: int):
        self.state = seed & MASK64

    def next_u64(self) -> int:
        self.state = (self.state + GOLDEN) & MASK64
        return mix64(self.state)

    def randint(self, lo: int, hi: int) -> int:
        """Uniform integer in [lo, hi] (inclusive)."""
        return lo + self.next_u64() % (hi - lo + 1)

    def permutation(self, n: int) -> np.ndarray:
        """Fisher-Yates shuffle of range(n)."""
        a = np.arange(n, dtype=np.int64)
        for i in range(n - 1, 0, -1):
            j = self.next_u64() % (i + 1)
            a[i], a[j] = a[j], a[i]
        return a


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (round to nearest, ties to even); uint16 bits."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    with np.errstate(over="ignore"):
        r = (b + np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _normal_chunk(key: int, start: int, n: int, sigma: float) -> np.ndarray:
    idx = np.arange(start, start + n, dtype=np.uint64)
    k = np.uint64(key)
    g = np.uint64(GOLDEN)
    with np.errstate(over="ignore"):
        z1 = _mix64_np(k + (np.uint64(2) * idx + np.uint64(1)) * g)
        z2 = _mix64_np(k + (np.uint64(2) * idx + np.uint64(2)) * g)
    u1 = ((z1 >> np.uint64(11)).astype(np.float64) + 1.0) * (2.0 ** -53)  # (0, 1]
    u2 = (z2 >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)  # [0, 1)
    x = np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * math.pi * u2)
    return f32_to_bf16_bits((x * sigma).astype(np.float32))


_CHUNK = 1 << 22
_POOL: Optional[ThreadPoolExecutor] = None


def _pool() -> ThreadPoolExecutor:
    global _POOL
    if _POOL is None:
        _POOL = ThreadPoolExecutor(max_workers=max(1, min(32, os.cpu_count() or 1)))
    return _POOL


def normal_bf16(key: int, start: int, n: int, sigma: float = 1.0) -> np.ndarray:
    """Elements [start, start+n) of the N(0, sigma^2) bf16 stream `key`."""
    if n <= _CHUNK:
        return _normal_chunk(key, start, n, sigma)
    out = np.empty(n, dtype=np.uint16)

    def work(off: int) -> None:
        m = min(_CHUNK, n - off)
        out[off:off + m] = _normal_chunk(key, start + off, m, sigma)

    list(_pool().map(work, range(0, n, _CHUNK)))
    return out


@dataclass
class Spec:
    """Shape and distribution of one workload."""

    name: str
    seed: int
    num_seqs: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    num_blocks: int
    sigma: float = 1.0
    # per-sequence context length at step 0, drawn uniform in [lo, hi]
    ctx_lo: int = 1
    ctx_hi: int = 1
    num_steps: int = 1
    # groups of `share_group` consecutive sequences share their first
    # `shared_blocks` physical blocks
    share_group: int = 0
    shared_blocks: int = 0
    # chunked-prefill mix: `prefill_seqs` sequences with `prefill_len` query rows
    # each and prior context uniform in [prior_lo, prior_hi]; the other
    # sequences decode (one query row)
    prefill_seqs: int = 0
    prefill_len: int = 0
    prior_lo: int = 0
    prior_hi: int = 0
    description: str = ""


@dataclass
class Workload:
    """A drawn workload: metadata on the host plus generators for contents."""

    spec: Spec
    ctx_lens0: np.ndarray  # int32 [B]: L_b at step 0 (tokens stored this step included)
    query_lens: np.ndarray  # int32 [B]: n_b, the same at every step
    seq_blocks: List[np.ndarray]  # physical block ids per sequence, in logical order
    max_blocks_per_seq: int
    _cache: Dict = field(default_factory=dict)

    # ---- shape shortcuts -------------------------------------------------
    @property
    def B(self) -> int:
        return self.spec.num_seqs

    @property
    def Hq(self) -> int:
        return self.spec.num_q_heads

    @property
    def Hkv(self) -> int:
        return self.spec.num_kv_heads

    @property
    def D(self) -> int:
        return self.spec.head_dim

    @property
    def BS(self) -> int:
        return self.spec.block_size

    @property
    def NB(self) -> int:
        return self.spec.num_blocks

    @property
    def total_q(self) -> int:
        return int(self.query_lens.sum())

    # ---- per-step metadata -----------------------------------------------
    def context_lens(self, step: int = 0) -> np.ndarray:
        return (self.ctx_lens0 + step * self.query_lens).astype(np.int32)

    def cu_seqlens_q(self) -> np.ndarray:
        cu = np.zeros(self.B + 1, dtype=np.int32)
        cu[1:] = np.cumsum(self.query_lens)
        return cu

    def block_tables(self, step: int = 0) -> np.ndarray:
        """[B, max_blocks_per_seq] int32; entries past the live blocks are -1."""
        L = self.context_lens(step)
        bt = np.full((self.B, self.max_blocks_per_seq), -1, dtype=np.int32)
        for b in range(self.B):
            nb = -(-int(L[b]) // self.BS)
            bt[b, :nb] = self.seq_blocks[b][:nb]
        return bt

    def token_positions(self, step: int = 0) -> Tuple[np.ndarray, np.ndarray]:
        """(seq index, absolute position) of every new token, packed by cu_seqlens_q."""
        L = self.context_lens(step)
        seq = np.repeat(np.arange(self.B, dtype=np.int64), self.query_lens)
        cu = self.cu_seqlens_q()
        row = np.arange(self.total_q, dtype=np.int64) - np.repeat(cu[:-1].astype(np.int64), self.query_lens)
        pos = np.repeat((L - self.query_lens).astype(np.int64), self.query_lens) + row
        return seq, pos

    def slot_mapping(self, step: int = 0) -> np.ndarray:
        """Cache slot of each new token: physical block id * block_size + offset."""
        seq, pos = self.token_positions(step)
        blk = np.array([self.seq_blocks[s][p // self.BS] for s, p in zip(seq, pos)], dtype=np.int64)
        return (blk * self.BS + pos % self.BS).astype(np.int32)

    # ---- contents ----------------------------------------------------------
    def q(self, step: int = 0) -> np.ndarray:
        """Query rows [total_q, Hq, D] as bf16 bits."""
        n = self.total_q * self.Hq * self.D
        return normal_bf16(stream_key(self.spec.seed, TAG_Q, step), 0, n, self.spec.sigma).reshape(
            self.total_q, self.Hq, self.D)

    def new_kv(self, step: int = 0) -> Tuple[np.ndarray, np.ndarray]:
        """Keys and values of this step's new tokens, [total_q, Hkv, D] bf16 bits.

        The token at absolute position j of sequence b always draws the same
        values, whichever step stores it.
        """
        hd = self.Hkv * self.D
        L = self.context_lens(step)
        ks, vs = [], []
        for b in range(self.B):
            n = int(self.query_lens[b])
            if n == 0:
                continue
            j0 = int(L[b]) - n
            ks.append(normal_bf16(stream_key(self.spec.seed, TAG_NEW_K, b), j0 * hd, n * hd, self.spec.sigma))
            vs.append(normal_bf16(stream_key(self.spec.seed, TAG_NEW_V, b), j0 * hd, n * hd, self.spec.sigma))
        k = np.concatenate(ks) if ks else np.zeros(0, np.uint16)
        v = np.concatenate(vs) if vs else np.zeros(0, np.uint16)
        return k.reshape(-1, self.Hkv, self.D), v.reshape(-1, self.Hkv, self.D)

    def prior_len(self, b: int) -> int:
        """Tokens already cached for sequence b before step 0's store."""
        return int(self.ctx_lens0[b]) - int(self.query_lens[b])

    def prior_fill(self) -> List[Tuple[int, int]]:
        """(physical block, number of leading slots holding cached tokens) before step 0."""
        valid: Dict[int, int] = {}
        for b in range(self.B):
            pl = self.prior_len(b)
            for i, p in enumerate(self.seq_blocks[b]):
                n = max(0, min(self.BS, pl - i * self.BS))
                if n > 0:
                    valid[int(p)] = max(valid.get(int(p), 0), n)
        return sorted(valid.items())

    def block_contents(self, p: int, n: int) -> Tuple[np.ndarray, np.ndarray]:
        """Cached keys/values of physical block p, slots [0, n): [n, Hkv, D] bf16 bits."""
        hd = self.Hkv * self.D
        k = normal_bf16(stream_key(self.spec.seed, TAG_POOL_K, p), 0, n * hd, self.spec.sigma)
        v = normal_bf16(stream_key(self.spec.seed, TAG_POOL_V, p), 0, n * hd, self.spec.sigma)
        return k.reshape(n, self.Hkv, self.D), v.reshape(n, self.Hkv, self.D)

    def prior_blocks_dense(self) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
        """All pre-filled blocks at once: (ids [U], K [U, BS, Hkv, D], V [U, BS, Hkv, D]).

        Slots past a block's cached prefix hold bf16 NaN.
        """
        fill = self.prior_fill()
        ids = np.array([p for p, _ in fill], dtype=np.int64)
        shape = (len(fill), self.BS, self.Hkv, self.D)
        K = np.full(shape, BF16_NAN, dtype=np.uint16)
        V = np.full(shape, BF16_NAN, dtype=np.uint16)
        for u, (p, n) in enumerate(fill):
            k, v = self.block_contents(p, n)
            K[u, :n] = k
            V[u, :n] = v
        return ids, K, V

    def host_pool(self) -> Tuple[np.ndarray, np.ndarray]:
        """Full [NB, BS, Hkv, D] pools as bf16 bits: NaN everywhere except cached tokens."""
        shape = (self.NB, self.BS, self.Hkv, self.D)
        kp = np.full(shape, BF16_NAN, dtype=np.uint16)
        vp = np.full(shape, BF16_NAN, dtype=np.uint16)
        ids, K, V = self.prior_blocks_dense()
        if len(ids):
            kp[ids] = K
            vp[ids] = V
        return kp, vp

    def kv_bytes_attended(self, step: int = 0) -> int:
        """K+V bytes a single pass over every sequence's live tokens reads."""
        return int(self.context_lens(step).astype(np.int64).sum()) * 2 * self.Hkv * self.D * 2

    def unique_kv_bytes(self, step: int = 0) -> int:
        """K+V bytes of distinct cache slots read (shared blocks counted once)."""
        L = self.context_lens(step)
        seen: Dict[int, int] = {}
        for b in range(self.B):
            for i, p in enumerate(self.seq_blocks[b]):
                n = max(0, min(self.BS, int(L[b]) - i * self.BS))
                if n:
                    seen[int(p)] = max(seen.get(int(p), 0), n)
        return sum(seen.values()) * 2 * self.Hkv * self.D * 2


def draw(spec: Spec) -> Workload:
    """Draw lengths and physical blocks for `spec` (deterministic in spec.seed)."""
    rng = SplitMix64(stream_key(spec.seed, TAG_META))
    B, BS = spec.num_seqs, spec.block_size
    qlen = np.ones(B, dtype=np.int32)
    ctx0 = np.zeros(B, dtype=np.int32)
    if spec.prefill_seqs:
        # which sequences prefill is itself drawn, so packing order is mixed
        order = rng.permutation(B)
        is_prefill = np.zeros(B, dtype=bool)
        is_prefill[order[: spec.prefill_seqs]] = True
        for b in range(B):
            if is_prefill[b]:
                qlen[b] = spec.prefill_len
                ctx0[b] = rng.randint(spec.prior_lo, spec.prior_hi) + spec.prefill_len
            else:
                ctx0[b] = rng.randint(spec.ctx_lo, spec.ctx_hi)
    else:
        for b in range(B):
            ctx0[b] = rng.randint(spec.ctx_lo, spec.ctx_hi)

    final = ctx0 + (spec.num_steps - 1) * qlen
    free = list(rng.permutation(spec.num_blocks))
    free.reverse()  # pop() takes from the front of the shuffled order

    def pop() -> int:
        if not free:
            raise ValueError(f"{spec.name}: block pool of {spec.num_blocks} exhausted")
        return int(free.pop())

    seq_blocks: List[List[int]] = [[] for _ in range(B)]
    shared: List[int] = []
    for b in range(B):
        need0 = -(-int(ctx0[b]) // BS)
        if spec.share_group and spec.shared_blocks:
            if b % spec.share_group == 0:
                shared = [pop() for _ in range(spec.shared_blocks)]
            if need0 <= spec.shared_blocks:
                raise ValueError("a shared block would receive new tokens")
            seq_blocks[b].extend(shared)
        while len(seq_blocks[b]) < need0:
            seq_blocks[b].append(pop())
    # blocks popped as decode steps cross block boundaries, step by step
    for step in range(1, spec.num_steps):
        L = ctx0 + step * qlen
        for b in range(B):
            while len(seq_blocks[b]) * BS < int(L[b]):
                seq_blocks[b].append(pop())
    mb = max(1, max(-(-int(f) // BS) for f in final))
    return Workload(spec=spec, ctx_lens0=ctx0, query_lens=qlen,
                    seq_blocks=[np.array(s, dtype=np.int64) for s in seq_blocks],
                    max_blocks_per_seq=mb)


# The named workloads.  `seed` is the workload's index.
SPECS: Dict[str, Spec] = {
    "tiny_decode": Spec(
        name="tiny_decode", seed=1, num_seqs=4, num_q_heads=4, num_kv_heads=2, head_dim=64,
        block_size=16, num_blocks=96, ctx_lo=1, ctx_hi=300,
        description="4 seqs, L~U[1,300], 4 Q / 2 KV heads, D=64, BS=16, 96-block shuffled pool; "
                    "store 1 token/seq then decode"),
    "qwen3_decode": Spec(
        name="qwen3_decode", seed=2, num_seqs=256, num_q_heads=16, num_kv_heads=8, head_dim=128,
        block_size=256, num_blocks=4096, ctx_lo=100, ctx_hi=2048, num_steps=64,
        description="Qwen3-0.6B-shaped decode: 256 seqs, L~U[100,2048], 16 Q / 8 KV heads, D=128, "
                    "BS=256, 4096-block shuffled pool; store 1 token/seq + decode, 64 steps"),
    "llama8b_prefix_decode": Spec(
        name="llama8b_prefix_decode", seed=3, num_seqs=64, num_q_heads=32, num_kv_heads=8, head_dim=128,
        block_size=256, num_blocks=4096, ctx_lo=4096, ctx_hi=8192, share_group=8, shared_blocks=8,
        description="LLaMA-8B-shaped GQA decode: 64 seqs, L~U[4096,8192], 32 Q / 8 KV heads, D=128, "
                    "BS=256; groups of 8 seqs share their first 8 physical blocks"),
    "long_context_decode": Spec(
        name="long_context_decode", seed=4, num_seqs=8, num_q_heads=32, num_kv_heads=8, head_dim=128,
        block_size=256, num_blocks=57344, sigma=0.5, ctx_lo=32768, ctx_hi=131072,
        description="long-context split-KV decode: 8 seqs, L~U[32768,131072], 32 Q / 8 KV heads, "
                    "D=128, BS=256, N(0,0.5^2); 57,344-block (~60 GB) pool"),
    "spec_verify_decode": Spec(
        name="spec_verify_decode", seed=6, num_seqs=256, num_q_heads=16, num_kv_heads=8, head_dim=128,
        block_size=256, num_blocks=4096, prefill_seqs=256, prefill_len=4, prior_lo=100, prior_hi=2044,
        description="speculative-decode verification: 256 seqs x 4 query rows (3 draft tokens + 1) "
                    "over prior context U[100,2044]; 16 Q / 8 KV heads, D=128, BS=256"),
    "chunked_prefill_mixed": Spec(
        name="chunked_prefill_mixed", seed=5, num_seqs=256, num_q_heads=16, num_kv_heads=8, head_dim=128,
        block_size=256, num_blocks=4096, ctx_lo=100, ctx_hi=2048, prefill_seqs=16, prefill_len=512,
        prior_lo=0, prior_hi=8192,
        description="chunked-prefill mixed batch: 16 seqs prefill a 512-token chunk over prior "
                    "context U[0,8192] + 240 decode seqs L~U[100,2048]; 16 Q / 8 KV heads, D=128, BS=256"),
}

# Headline workload for throughput reporting.
HEADLINE = "qwen3_decode"

# Smaller variants of the same shapes, for profiler captures that must stay a
# few GB on the device (the KV read per launch still exceeds the 126 MB L2).
PROFILE_SPECS: Dict[str, Spec] = {
    "qwen3_decode_small": Spec(
        name="qwen3_decode_small", seed=2, num_seqs=64, num_q_heads=16, num_kv_heads=8, head_dim=128,
        block_size=256, num_blocks=1024, ctx_lo=100, ctx_hi=2048, num_steps=4,
        description="qwen3_decode with 64 sequences and a 1,024-block pool (profiling size)"),
    "chunked_prefill_small": Spec(
        name="chunked_prefill_small", seed=5, num_seqs=32, num_q_heads=16, num_kv_heads=8, head_dim=128,
        block_size=256, num_blocks=1024, ctx_lo=100, ctx_hi=2048, prefill_seqs=16, prefill_len=512,
        prior_lo=0, prior_hi=8192,
        description="chunked_prefill_mixed with all 16 prefill sequences but 16 decode sequences and a "
                    "1,024-block pool (profiling size: 1 GB of cache on the device)"),
}


def workload(name: str) -> Workload:
    return draw(SPECS[name] if name in SPECS else PROFILE_SPECS[name])


def scaled(spec: Spec, **changes) -> Spec:
    """A copy of `spec` with some fields replaced (for smaller test variants)."""
    d = dict(spec.__dict__)
    d.update(changes)
    return Spec(**d)


# ---------------------------------------------------------------------------
# Device copies (torch supplies the memory; nothing here computes attention)
# ---------------------------------------------------------------------------

def bits_to_torch(a: np.ndarray, device=None):
    """uint16 bf16 bit patterns -> torch.bfloat16 tensor (same bits)."""
    import torch

    t = torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)
    return t.to(device) if device is not None else t


def torch_to_bits(t) -> np.ndarray:
    """torch.bfloat16 tensor -> uint16 numpy array of its bit patterns."""
    import torch

    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


class DeviceState:
    """A workload's cache and per-step inputs resident on one CUDA device.

    The caches are [NB, BS, Hkv, D] bf16, filled with bf16 NaN except the cached
    prefix of every sequence, so any read outside a sequence's live tokens shows
    up as NaN in the output.
    """

    def __init__(self, wl: Workload, device, steps: Optional[List[int]] = None):
        import torch

        self.wl = wl
        self.device = torch.device(device)
        shape = (wl.NB, wl.BS, wl.Hkv, wl.D)
        self.k_cache = torch.empty(shape, dtype=torch.bfloat16, device=self.device)
        self.v_cache = torch.empty(shape, dtype=torch.bfloat16, device=self.device)
        nan = int(np.int16(np.uint16(BF16_NAN).view(np.int16)))
        self.k_cache.view(torch.int16).fill_(nan)
        self.v_cache.view(torch.int16).fill_(nan)
        ids, K, V = wl.prior_blocks_dense()
        if len(ids):
            idx = torch.from_numpy(ids).to(self.device)
            # copy in slices to bound the host->device staging footprint
            step = max(1, (1 << 28) // max(1, K[0].nbytes))
            for s in range(0, len(ids), step):
                self.k_cache.index_copy_(0, idx[s:s + step], bits_to_torch(K[s:s + step], self.device))
                self.v_cache.index_copy_(0, idx[s:s + step], bits_to_torch(V[s:s + step], self.device))
        del K, V
        self.steps = {}
        for st in (steps if steps is not None else [0]):
            self.steps[st] = self.step_inputs(st)

    def step_inputs(self, step: int) -> Dict[str, "object"]:
        import torch

        wl = self.wl
        d = self.device
        k, v = wl.new_kv(step)
        return {
            "q": bits_to_torch(wl.q(step), d),
            "key": bits_to_torch(k, d),
            "value": bits_to_torch(v, d),
            "slot_mapping": torch.from_numpy(wl.slot_mapping(step)).to(d),
            "block_tables": torch.from_numpy(wl.block_tables(step)).to(d),
            "context_lens": torch.from_numpy(wl.context_lens(step)).to(d),
            "cu_seqlens_q": torch.from_numpy(wl.cu_seqlens_q()).to(d),
            "max_seqlen_q": int(wl.query_lens.max()) if wl.B else 0,
        }
