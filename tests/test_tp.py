"""Head-sharded decode attention with the o_proj all-reduce: the host logic on CPU.

Two gloo ranks each take half of the KV heads (and their query heads), compute
their heads' attention (here with the fp64 oracle, rounded to bf16 as the
kernels' output is), multiply by their slice of W_o and all-reduce.  Both ranks
must end with the same output, equal to the unsharded o_proj of all heads
within the rounding bound of tests/tp_cases.py.  The row-parallel split is the
block identity sum_r A_r W_r^T = A W^T ("Nano-vLLM Architecture and Performance",
Key Features 3: the projections are sharded along the head dimension).
"""

import datetime
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from paged_kv_cache_bf16_b200 import tp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.mark.parametrize("hq,hkv,world", [(16, 8, 1), (16, 8, 2), (32, 8, 4), (8, 8, 8), (64, 8, 2), (4, 2, 2)])
def test_shards_partition_heads_and_keep_gqa_groups(hq, hkv, world):
    g = hq // hkv
    seen_q, seen_kv = [], []
    for r in range(world):
        s = tp.shard_heads(hq, hkv, world, r)
        assert s.num_kv_heads == hkv // world and s.num_q_heads == hq // world
        seen_kv += list(range(s.kv0, s.kv1))
        seen_q += list(range(s.q0, s.q1))
        for h in range(s.q0, s.q1):
            assert s.kv0 <= h // g < s.kv1  # a query head's KV head lives on its rank
    assert seen_q == list(range(hq)) and seen_kv == list(range(hkv))


def test_shard_rejects_uneven_splits():
    with pytest.raises(ValueError):
        tp.shard_heads(16, 8, 3, 0)
    with pytest.raises(ValueError):
        tp.shard_heads(12, 8, 2, 0)
    with pytest.raises(ValueError):
        tp.shard_heads(16, 8, 2, 2)


def test_local_slices():
    s = tp.shard_heads(16, 8, 4, 2)
    q = torch.arange(3 * 16 * 4).reshape(3, 16, 4)
    kv = torch.arange(3 * 8 * 4).reshape(3, 8, 4)
    pool = torch.arange(5 * 2 * 8 * 4).reshape(5, 2, 8, 4)
    w = torch.arange(7 * 16 * 4).reshape(7, 64)
    assert torch.equal(tp.local_q(q, s), q[:, 8:12])
    assert torch.equal(tp.local_kv(kv, s), kv[:, 4:6])
    assert torch.equal(tp.local_kv(pool, s), pool[:, :, 4:6])
    assert torch.equal(tp.local_oproj_weight(w, s, 4), w[:, 32:48])


def _free_port() -> int:
    so = socket.socket()
    so.bind(("127.0.0.1", 0))
    port = so.getsockname()[1]
    so.close()
    return port


def _rank_main(rank, world, port, attn_bits, w_bits, hq, hkv, d, q):
    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    sys.path.insert(0, HERE)
    from paged_kv_cache_bf16_b200 import tp as TP

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        s = TP.shard_heads(hq, hkv, world, rank)
        attn = torch.from_numpy(attn_bits.view(np.int16)).view(torch.bfloat16)
        w = torch.from_numpy(w_bits.view(np.int16)).view(torch.bfloat16)
        a_loc = TP.local_q(attn, s)
        w_loc = TP.local_oproj_weight(w, s, d)
        partial = TP.oproj_partial(a_loc, w_loc).double().numpy()
        y = TP.oproj_allreduce(a_loc, w_loc)
        q.put((rank, y.view(torch.int16).numpy().view(np.uint16), np.abs(partial)))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_gloo_ranks_oproj_allreduce_matches_unsharded(world):
    from oracle import oracle as O
    from cases import oracle_post_store
    from tp_cases import HIDDEN, oproj_bound, oproj_weight, tp_workload

    wl = tp_workload()
    kp, vp = oracle_post_store(wl)
    attn64 = O.decode_attention(wl.q(0), kp, vp, wl.block_tables(0), wl.context_lens(0))
    attn_bits = O.to_bf16(attn64)  # the kernels' output is bf16
    K = wl.Hq * wl.D
    w_bits = oproj_weight(8101, HIDDEN, K)
    a = O.bf16_to_f64(attn_bits).reshape(wl.B, K)
    wf = O.bf16_to_f64(w_bits)
    y_ref = a @ wf.T

    ctx = mp.get_context("spawn")
    qu = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, attn_bits, w_bits, wl.Hq, wl.Hkv, wl.D, qu))
             for r in range(world)]
    for p in procs:
        p.start()
    res = sorted([qu.get(timeout=120) for _ in range(world)], key=lambda x: x[0])
    for p in procs:
        p.join(60)
        assert p.exitcode == 0
    ys = [r[1] for r in res]
    for y in ys[1:]:
        assert np.array_equal(y, ys[0])  # every rank holds the same output
    partial_abs = sum(r[2] for r in res)
    err = np.abs(O.bf16_to_f64(ys[0]) - y_ref)
    bound = oproj_bound(a, wf, partial_abs, y_ref)
    assert (err <= bound).all(), float((err - bound).max())
    # the row-parallel sum is not a no-op: each rank's share is a large part of y
    assert np.median(partial_abs) > 0.1 * np.median(np.abs(y_ref))
