"""Head-sharded (tensor-parallel) decode attention with the o_proj all-reduce.

"Nano-vLLM Architecture and Performance", Key Features 3 (Tensor Parallelism):
the QKV and output projections are sharded along the head dimension across
GPUs, one process per GPU.  The output projection is row-parallel: each rank
multiplies its own heads' attention output by its slice of W_o's input
columns, and the per-rank partial products are summed across ranks.

Layout per rank: the rank owns a contiguous range of KV heads and the g query
heads of each (GQA groups are never split), keeps the KV pool of those heads
only ([num_blocks, block_size, Hkv / world, D] in its own HBM), and runs the
library's ordinary fused store + decode call on them; nothing crosses between
GPUs until the o_proj partial sums, whose all-reduce is the step's one
collective (NCCL over NVLink on GPUs, gloo on CPU).  The partial products are
reduced in fp32 and rounded to bf16 once.
"""

from __future__ import annotations

from dataclasses import dataclass
from typing import Optional

import torch
import torch.distributed as dist

from . import ops


@dataclass(frozen=True)
class HeadShard:
    """Heads owned by `rank` of `world`: KV heads [kv0, kv1), query heads [q0, q1)."""

    rank: int
    world: int
    kv0: int
    kv1: int
    q0: int
    q1: int

    @property
    def num_kv_heads(self) -> int:
        return self.kv1 - self.kv0

    @property
    def num_q_heads(self) -> int:
        return self.q1 - self.q0


def shard_heads(num_q_heads: int, num_kv_heads: int, world: int, rank: int) -> HeadShard:
    """Contiguous, equal head ranges: rank r owns KV heads [r Hkv/w, (r+1) Hkv/w) and
    their query heads (query head h reads KV head h / g, so those are consecutive)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} of world {world}")
    if num_kv_heads <= 0 or num_q_heads % num_kv_heads != 0:
        raise ValueError(f"{num_q_heads} query heads over {num_kv_heads} KV heads")
    if num_kv_heads % world != 0:
        raise ValueError(f"{num_kv_heads} KV heads do not split over {world} ranks")
    g = num_q_heads // num_kv_heads
    per = num_kv_heads // world
    kv0 = rank * per
    return HeadShard(rank, world, kv0, kv0 + per, kv0 * g, (kv0 + per) * g)


def local_q(x: torch.Tensor, shard: HeadShard) -> torch.Tensor:
    """This rank's query heads of [T, Hq, D] rows."""
    return x[:, shard.q0:shard.q1].contiguous()


def local_kv(x: torch.Tensor, shard: HeadShard) -> torch.Tensor:
    """This rank's KV heads of [T, Hkv, D] rows or of a [NB, BS, Hkv, D] pool."""
    return x[..., shard.kv0:shard.kv1, :].contiguous()


def local_oproj_weight(w_o: torch.Tensor, shard: HeadShard, head_dim: int) -> torch.Tensor:
    """Input columns of W_o [hidden, Hq * D] that this rank's heads feed."""
    return w_o[:, shard.q0 * head_dim:shard.q1 * head_dim].contiguous()


def oproj_partial(attn_local: torch.Tensor, w_o_local: torch.Tensor) -> torch.Tensor:
    """This rank's share of o_proj: attn [T, Hq_local, D] (bf16) times the local
    W_o columns [hidden, Hq_local * D]; fp32 [T, hidden]."""
    T = attn_local.shape[0]
    return torch.matmul(attn_local.reshape(T, -1), w_o_local.t()).float()


def oproj_allreduce(attn_local: torch.Tensor, w_o_local: torch.Tensor, group=None) -> torch.Tensor:
    """Row-parallel o_proj: the local partial product, summed over the ranks of
    `group` (fp32), rounded to bf16.  [T, hidden]."""
    y = oproj_partial(attn_local, w_o_local)
    if dist.is_initialized():
        dist.all_reduce(y, op=dist.ReduceOp.SUM, group=group)
    return y.to(torch.bfloat16)


class TPDecodeLayer:
    """One attention layer's decode step on this rank's heads.

    k_cache / v_cache hold only this rank's KV heads; w_o_local is this rank's
    slice of W_o (local_oproj_weight).  step() stores the new tokens' K/V rows,
    attends over the paged cache (npv_store_kvcache_and_decode_attention) and
    returns the full o_proj output [B, hidden] bf16, identical on every rank.
    """

    def __init__(self, shard: HeadShard, k_cache: torch.Tensor, v_cache: torch.Tensor, w_o_local: torch.Tensor,
                 group=None):
        if k_cache.shape[2] != shard.num_kv_heads:
            raise ValueError(f"cache holds {k_cache.shape[2]} KV heads, the shard {shard.num_kv_heads}")
        D = k_cache.shape[3]
        if w_o_local.shape[1] != shard.num_q_heads * D:
            raise ValueError(f"W_o slice has {w_o_local.shape[1]} input columns, expected {shard.num_q_heads * D}")
        self.shard = shard
        self.k_cache = k_cache
        self.v_cache = v_cache
        self.w_o_local = w_o_local
        self.group = group
        self._ws: Optional[torch.Tensor] = None

    def step(self, q_local: torch.Tensor, key_local: torch.Tensor, value_local: torch.Tensor,
             slot_mapping: torch.Tensor, block_tables: torch.Tensor, context_lens: torch.Tensor) -> torch.Tensor:
        B = q_local.shape[0]
        D = self.k_cache.shape[3]
        need = ops.decode_workspace_size(B, self.shard.num_q_heads, self.shard.num_kv_heads, D)
        if self._ws is None or self._ws.numel() < need:
            self._ws = ops.alloc_workspace(need, q_local.device)
        attn = ops.store_kvcache_and_decode_attention(q_local, key_local, value_local, self.k_cache, self.v_cache,
                                                      slot_mapping, block_tables, context_lens, workspace=self._ws)
        return oproj_allreduce(attn, self.w_o_local, self.group)
