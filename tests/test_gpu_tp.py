"""Head-sharded decode attention with the o_proj all-reduce on the GPU.

This run has one GPU, so the collective runs as a one-rank NCCL group (the
kernels, the o_proj GEMM and NCCL's all-reduce all on the device), and the
two-rank split runs its shards one after the other on the same GPU with the sum
taken on the host (no rank ever waits for another).  Attention is checked
against the fp64 oracle at the attention tolerance; the o_proj output against
the fp64 product of the kernels' own bf16 attention output and W_o, within the
rounding bound of tests/tp_cases.py.  Not measured across GPUs.
"""

import datetime
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

from cases import oracle_post_store
from gpu_common import DEV, assert_close, no_device_errors, out_f64
from oracle import oracle as O
from paged_kv_cache_bf16_b200 import ops, tp
from paged_kv_cache_bf16_b200 import workloads as W
from tp_cases import HIDDEN, oproj_bound, oproj_weight, tp_workload

pytestmark = pytest.mark.gpu


def _free_port() -> int:
    so = socket.socket()
    so.bind(("127.0.0.1", 0))
    port = so.getsockname()[1]
    so.close()
    return port


def _w(wl, seed):
    bits = oproj_weight(seed, HIDDEN, wl.Hq * wl.D)
    return bits, torch.from_numpy(bits.view(np.int16)).to(DEV).view(torch.bfloat16)


def _check_oproj(y, a_gpu, w_bits, partials_abs):
    a = out_f64(a_gpu).reshape(a_gpu.shape[0], -1)
    wf = O.bf16_to_f64(w_bits)
    y_ref = a @ wf.T
    err = np.abs(out_f64(y) - y_ref)
    bound = oproj_bound(a, wf, partials_abs, y_ref)
    assert (err <= bound).all(), float((err - bound).max())


def test_one_rank_nccl_layer():
    wl = tp_workload(seed=8200)
    st = W.DeviceState(wl, DEV)
    s = st.steps[0]
    w_bits, w = _w(wl, 8201)
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60))
    try:
        shard = tp.shard_heads(wl.Hq, wl.Hkv, 1, 0)
        layer = tp.TPDecodeLayer(shard, st.k_cache, st.v_cache, tp.local_oproj_weight(w, shard, wl.D))
        y = layer.step(s["q"], s["key"], s["value"], s["slot_mapping"], s["block_tables"], s["context_lens"])
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    no_device_errors()
    # the step's attention, read again from the cache it stored into
    a = ops.paged_decode_attention(s["q"], st.k_cache, st.v_cache, s["block_tables"], s["context_lens"])
    kp, vp = oracle_post_store(wl)
    assert_close(a, O.decode_attention(wl.q(0), kp, vp, wl.block_tables(0), wl.context_lens(0)), "attention")
    partial = np.abs(out_f64(a).reshape(wl.B, -1) @ O.bf16_to_f64(w_bits).T)
    _check_oproj(y, a, w_bits, partial)


@pytest.mark.parametrize("hq,hkv,world", [(16, 8, 2), (32, 8, 4)])
def test_shards_one_after_another_sum_to_unsharded(hq, hkv, world):
    wl = tp_workload(seed=8300 + world, hq=hq, hkv=hkv)
    st = W.DeviceState(wl, DEV)
    s = st.steps[0]
    w_bits, w = _w(wl, 8301)
    attn, partials = [], []
    for r in range(world):
        sh = tp.shard_heads(wl.Hq, wl.Hkv, world, r)
        kc, vc = tp.local_kv(st.k_cache, sh), tp.local_kv(st.v_cache, sh)
        a_r = ops.store_kvcache_and_decode_attention(tp.local_q(s["q"], sh), tp.local_kv(s["key"], sh),
                                                     tp.local_kv(s["value"], sh), kc, vc, s["slot_mapping"],
                                                     s["block_tables"], s["context_lens"])
        attn.append(a_r)
        partials.append(tp.oproj_partial(a_r, tp.local_oproj_weight(w, sh, wl.D)))
    no_device_errors()
    y = torch.stack(partials).sum(0).to(torch.bfloat16)
    a = torch.cat(attn, dim=1)
    kp, vp = oracle_post_store(wl)
    assert_close(a, O.decode_attention(wl.q(0), kp, vp, wl.block_tables(0), wl.context_lens(0)), "sharded attention")
    _check_oproj(y, a, w_bits, sum(np.abs(out_f64(p)) for p in partials))
