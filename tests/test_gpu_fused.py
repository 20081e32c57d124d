"""npv_store_kvcache_and_decode_attention: bit-identical to store then decode (GPU)."""

import numpy as np
import pytest
import torch

from cases import oracle_compact, tiny_spec
from gpu_common import DEV, assert_close, no_device_errors, run_decode, run_store
from paged_kv_cache_bf16_b200 import ops
from paged_kv_cache_bf16_b200 import workloads as W

pytestmark = pytest.mark.gpu


def fused(st, step, **kw):
    s = st.steps[step]
    return ops.store_kvcache_and_decode_attention(s["q"], s["key"], s["value"], st.k_cache, st.v_cache,
                                                  s["slot_mapping"], s["block_tables"], s["context_lens"], **kw)


SPECS = {
    "tiny_decode": W.SPECS["tiny_decode"],
    "qwen3_like": tiny_spec(name="f_qwen", seed=901, head_dim=128, num_q_heads=16, num_kv_heads=8, block_size=256,
                            num_blocks=300, num_seqs=40, ctx_lo=1, ctx_hi=2048),
    "two_head_groups": tiny_spec(name="f_hkv16", seed=902, head_dim=128, num_q_heads=32, num_kv_heads=16,
                                 block_size=32, num_blocks=400, num_seqs=9, ctx_lo=1, ctx_hi=900),
    "g4_d64": tiny_spec(name="f_g4", seed=903, head_dim=64, num_q_heads=16, num_kv_heads=4, block_size=16,
                        num_blocks=500, num_seqs=12, ctx_lo=1, ctx_hi=500),
    "prefix": tiny_spec(name="f_prefix", seed=904, head_dim=128, num_q_heads=32, num_kv_heads=8, block_size=256,
                        num_blocks=200, num_seqs=16, ctx_lo=1100, ctx_hi=3000, share_group=4, shared_blocks=4),
}


@pytest.mark.parametrize("name", sorted(SPECS))
def test_fused_equals_store_then_decode(name):
    wl = W.draw(SPECS[name])
    a = W.DeviceState(wl, DEV)
    b = W.DeviceState(wl, DEV)
    run_store(a, 0)
    ref = run_decode(a, 0)
    out = fused(b, 0)
    no_device_errors()
    assert torch.equal(out.view(torch.int16), ref.view(torch.int16))
    assert torch.equal(a.k_cache.view(torch.int16), b.k_cache.view(torch.int16))
    assert torch.equal(a.v_cache.view(torch.int16), b.v_cache.view(torch.int16))
    oref, _ = oracle_compact(wl, 0)
    assert_close(out, oref, name)


def test_fused_qwen3_decode_64_steps():
    wl = W.workload("qwen3_decode")
    st = W.DeviceState(wl, DEV, steps=list(range(wl.spec.num_steps)))
    keep = {}
    for step in range(wl.spec.num_steps):
        out = fused(st, step)
        if step in (0, 63):
            keep[step] = out.clone()
    no_device_errors()
    for step, out in keep.items():
        ref, rows = oracle_compact(wl, step)
        assert_close(out[torch.from_numpy(rows).to(DEV)], ref, f"step {step}")


def test_fused_padding_zero_length_and_negative_slots():
    wl = W.draw(SPECS["qwen3_like"])
    a = W.DeviceState(wl, DEV)
    b = W.DeviceState(wl, DEV)
    s = a.steps[0]
    cl = s["context_lens"].clone()
    slots = s["slot_mapping"].clone()
    cl[3] = 0          # a padding sequence whose token is still stored
    slots[5] = -1      # a token that is not stored
    ops.store_kvcache(s["key"], s["value"], a.k_cache, a.v_cache, slots)
    ref = ops.paged_decode_attention(s["q"], a.k_cache, a.v_cache, s["block_tables"], cl)
    out = ops.store_kvcache_and_decode_attention(s["q"], s["key"], s["value"], b.k_cache, b.v_cache, slots,
                                                 s["block_tables"], cl)
    no_device_errors()
    assert torch.equal(out.view(torch.int16), ref.view(torch.int16))
    assert torch.count_nonzero(out[3]).item() == 0
    assert torch.equal(a.k_cache.view(torch.int16), b.k_cache.view(torch.int16))
    assert torch.equal(a.v_cache.view(torch.int16), b.v_cache.view(torch.int16))
