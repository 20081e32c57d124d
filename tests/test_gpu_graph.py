"""Decode steps captured in one CUDA graph and replayed give the eager calls'
bits, and both match the fp64 oracle step by step (GPU).  The library's launches
(programmatic dependent launch between the split-KV and merge kernels) are
capturable once a first eager call has set the kernels' shared-memory limits."""

import pytest
import torch

from cases import oracle_compact, tiny_spec
from gpu_common import DEV, assert_close, no_device_errors
from paged_kv_cache_bf16_b200 import ops
from paged_kv_cache_bf16_b200 import workloads as W

pytestmark = pytest.mark.gpu

NSTEPS = 6


def _steps(st, wl, outs, ws, fused=True):
    for i in range(NSTEPS):
        s = st.steps[i]
        if fused:
            ops.store_kvcache_and_decode_attention(s["q"], s["key"], s["value"], st.k_cache, st.v_cache,
                                                   s["slot_mapping"], s["block_tables"], s["context_lens"],
                                                   out=outs[i], workspace=ws)
        else:
            # store -> split -> merge -> store ...: every launch chained by
            # programmatic dependent launch, the store waiting on the merge before it
            ops.store_kvcache(s["key"], s["value"], st.k_cache, st.v_cache, s["slot_mapping"])
            ops.paged_decode_attention(s["q"], st.k_cache, st.v_cache, s["block_tables"], s["context_lens"],
                                       out=outs[i], workspace=ws)


@pytest.mark.parametrize("hq,hkv,bs,fused", [(16, 8, 256, True), (32, 8, 16, True), (16, 8, 256, False)])
def test_decode_steps_from_a_cuda_graph_match_eager(hq, hkv, bs, fused):
    spec = tiny_spec(name="graph", seed=901 + hq, head_dim=128, num_q_heads=hq, num_kv_heads=hkv, block_size=bs,
                     num_blocks=2000 if bs == 16 else 200, num_seqs=24, ctx_lo=1, ctx_hi=900, num_steps=NSTEPS)
    wl = W.draw(spec)
    ws_bytes = ops.decode_workspace_size(wl.B, wl.Hq, wl.Hkv, wl.D)

    eager = W.DeviceState(wl, DEV, steps=list(range(NSTEPS)))
    outs_e = [torch.empty((wl.B, wl.Hq, wl.D), dtype=torch.bfloat16, device=DEV) for _ in range(NSTEPS)]
    _steps(eager, wl, outs_e, ops.alloc_workspace(ws_bytes, DEV), fused)
    no_device_errors()

    replay = W.DeviceState(wl, DEV, steps=list(range(NSTEPS)))
    outs_g = [torch.empty_like(o) for o in outs_e]
    ws = ops.alloc_workspace(ws_bytes, DEV)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        _steps(replay, wl, outs_g, ws, fused)
    g.replay()
    torch.cuda.synchronize()
    no_device_errors()
    for i in range(NSTEPS):
        assert torch.equal(outs_g[i].view(torch.int16), outs_e[i].view(torch.int16)), f"step {i}"
    assert torch.equal(replay.k_cache.view(torch.int16), eager.k_cache.view(torch.int16))
    assert torch.equal(replay.v_cache.view(torch.int16), eager.v_cache.view(torch.int16))
    # every replayed step against the oracle (stores of steps 0..i applied by the oracle)
    for i in range(NSTEPS):
        ref, rows = oracle_compact(wl, i)
        assert_close(outs_g[i][torch.from_numpy(rows).to(DEV)], ref, f"graph step {i}")
    # a second replay repeats the same stores and the same results
    g.replay()
    torch.cuda.synchronize()
    for i in range(NSTEPS):
        assert torch.equal(outs_g[i].view(torch.int16), outs_e[i].view(torch.int16)), f"replay 2 step {i}"
