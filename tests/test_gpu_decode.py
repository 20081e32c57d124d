"""npv_paged_decode_attention against the fp64 oracle (GPU).

Inputs are the seeded workloads (shapes of the pages' engine); every pool slot
outside a sequence's live tokens is bf16 NaN, so a stray read fails the test.
Tolerance: max-abs 1.5e-2 and mean-abs 2e-3 against fp64.
"""

import numpy as np
import pytest
import torch

from cases import oracle_compact, tiny_spec
from gpu_common import DEV, assert_close, no_device_errors, run_decode, run_store
from paged_kv_cache_bf16_b200 import ops
from paged_kv_cache_bf16_b200 import workloads as W

pytestmark = pytest.mark.gpu

DECODE_NAMED = ["tiny_decode", "qwen3_decode", "llama8b_prefix_decode", "long_context_decode"]


@pytest.mark.parametrize("name", DECODE_NAMED)
def test_decode_named_workload(name):
    wl = W.workload(name)
    st = W.DeviceState(wl, DEV)
    run_store(st, 0)
    out = run_decode(st, 0)
    no_device_errors()
    ref, rows = oracle_compact(wl, 0)
    assert_close(out[torch.from_numpy(rows).to(DEV)], ref, name)
    del st
    torch.cuda.empty_cache()


def test_qwen3_decode_64_steps():
    """64 store + decode steps; blocks are popped as sequences cross block boundaries."""
    wl = W.workload("qwen3_decode")
    check = {0: None, 1: None, 37: None, 63: None}
    st = W.DeviceState(wl, DEV, steps=list(range(wl.spec.num_steps)))
    for step in range(wl.spec.num_steps):
        run_store(st, step)
        out = run_decode(st, step)
        if step in check:
            check[step] = out.clone()
    no_device_errors()
    for step, out in check.items():
        ref, rows = oracle_compact(wl, step)
        assert_close(out[torch.from_numpy(rows).to(DEV)], ref, f"step {step}")


SHAPES = [
    # (head_dim, Hq, Hkv, block_size, ctx_hi, num_seqs)
    (64, 4, 2, 16, 300, 4),
    (64, 8, 8, 16, 500, 6),
    (64, 16, 2, 32, 700, 5),
    (64, 32, 4, 64, 900, 3),
    (128, 8, 8, 16, 400, 7),
    (128, 16, 8, 256, 3000, 9),
    (128, 32, 8, 256, 2000, 5),
    (128, 64, 8, 256, 1500, 3),
    (128, 16, 16, 32, 600, 4),
    (128, 8, 1, 48, 800, 6),
    (128, 4, 4, 128, 5000, 2),
]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "D%d_q%d_kv%d_bs%d_L%d_B%d" % s)
def test_decode_shapes(shape):
    D, Hq, Hkv, BS, hi, B = shape
    nb = B * (-(-hi // BS)) + 8
    spec = tiny_spec(seed=1000 + sum(shape), head_dim=D, num_q_heads=Hq, num_kv_heads=Hkv, block_size=BS,
                     num_blocks=nb, num_seqs=B, ctx_lo=1, ctx_hi=hi)
    wl = W.draw(spec)
    st = W.DeviceState(wl, DEV)
    run_store(st, 0)
    out = run_decode(st, 0)
    no_device_errors()
    ref, rows = oracle_compact(wl, 0)
    assert_close(out, ref, str(shape))


def _fixed_lengths_spec(lengths, **kw):
    spec = tiny_spec(seed=77, head_dim=128, num_q_heads=16, num_kv_heads=8, block_size=256,
                     num_blocks=sum(-(-L // 256) for L in lengths) + 4, num_seqs=len(lengths), **kw)
    return spec


def _with_lengths(spec, lengths):
    wl = W.draw(spec)
    L = np.array(lengths, dtype=np.int32)
    # redraw block lists for the fixed lengths from the same shuffled pool
    perm = list(W.SplitMix64(spec.seed).permutation(spec.num_blocks))
    blocks = []
    for b in range(len(L)):
        n = -(-int(L[b]) // spec.block_size)
        blocks.append(np.array([perm.pop() for _ in range(n)], dtype=np.int64))
    return W.Workload(spec=spec, ctx_lens0=L, query_lens=np.ones(len(L), np.int32), seq_blocks=blocks,
                      max_blocks_per_seq=max(len(x) for x in blocks))


def test_decode_context_length_edges():
    lengths = [1, 2, 15, 16, 17, 31, 32, 33, 255, 256, 257, 511, 512, 513, 1000, 4095, 4096, 4097]
    wl = _with_lengths(_fixed_lengths_spec(lengths), lengths)
    st = W.DeviceState(wl, DEV)
    run_store(st, 0)
    out = run_decode(st, 0)
    no_device_errors()
    ref, rows = oracle_compact(wl, 0)
    assert_close(out, ref, "edges")


def test_one_token_context_returns_v_exactly():
    lengths = [1] * 37
    wl = _with_lengths(_fixed_lengths_spec(lengths), lengths)
    st = W.DeviceState(wl, DEV)
    run_store(st, 0)
    out = run_decode(st, 0)
    no_device_errors()
    _, v = wl.new_kv(0)  # [B, Hkv, D]; query head h reads KV head h // g
    g = wl.Hq // wl.Hkv
    expect = np.repeat(v, g, axis=1)
    assert np.array_equal(W.torch_to_bits(out), expect)


def test_zero_length_rows_are_zero_and_invalid_lengths_reported():
    lengths = [5, 300, 7]
    wl = _with_lengths(_fixed_lengths_spec(lengths), lengths)
    st = W.DeviceState(wl, DEV)
    run_store(st, 0)
    s = st.steps[0]
    cl = s["context_lens"].clone()
    cl[1] = 0
    out = ops.paged_decode_attention(s["q"], st.k_cache, st.v_cache, s["block_tables"], cl)
    assert ops.check_device_errors() == 0
    assert torch.count_nonzero(out[1]).item() == 0
    cl[1] = wl.max_blocks_per_seq * wl.BS + 1
    out = ops.paged_decode_attention(s["q"], st.k_cache, st.v_cache, s["block_tables"], cl)
    with pytest.raises(ops.NpvError) as ei:
        ops.check_device_errors()
    assert ei.value.bits & 0x4
    assert torch.count_nonzero(out[1]).item() == 0
    ref, rows = oracle_compact(wl, 0, seqs=[0, 2])
    assert_close(out[[0, 2]], ref, "other rows")


def test_invalid_block_id_is_reported_not_faulted():
    wl = W.draw(tiny_spec(seed=5, head_dim=128, num_q_heads=16, num_kv_heads=8, block_size=16, num_blocks=300,
                          num_seqs=6, ctx_lo=40, ctx_hi=200))
    st = W.DeviceState(wl, DEV)
    run_store(st, 0)
    s = st.steps[0]
    bt = s["block_tables"].clone()
    bt[2, 1] = wl.NB + 5
    bt[4, 0] = -3
    ops.paged_decode_attention(s["q"], st.k_cache, st.v_cache, bt, s["context_lens"])
    with pytest.raises(ops.NpvError) as ei:
        ops.check_device_errors()
    assert ei.value.bits & 0x2
    out = run_decode(st, 0)  # the context is still usable
    no_device_errors()
    ref, _ = oracle_compact(wl, 0)
    assert_close(out, ref, "after error")


def test_relabelled_blocks_give_identical_bits():
    wl = W.workload("tiny_decode")
    st = W.DeviceState(wl, DEV)
    run_store(st, 0)
    out = run_decode(st, 0)
    perm = torch.from_numpy(np.random.default_rng(3).permutation(wl.NB)).to(DEV)
    k2 = torch.empty_like(st.k_cache)
    v2 = torch.empty_like(st.v_cache)
    k2[perm] = st.k_cache
    v2[perm] = st.v_cache
    s = st.steps[0]
    bt = s["block_tables"]
    bt2 = torch.where(bt >= 0, perm[bt.clamp(min=0).long()].int(), bt)
    out2 = ops.paged_decode_attention(s["q"], k2, v2, bt2, s["context_lens"])
    no_device_errors()
    assert torch.equal(out.view(torch.int16), out2.view(torch.int16))


def test_decode_deterministic_and_explicit_scale():
    wl = W.draw(tiny_spec(seed=8, head_dim=128, num_q_heads=32, num_kv_heads=8, block_size=256, num_blocks=80,
                          num_seqs=12, ctx_lo=100, ctx_hi=1500))
    st = W.DeviceState(wl, DEV)
    run_store(st, 0)
    a = run_decode(st, 0)
    b = run_decode(st, 0)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    c = run_decode(st, 0, scale=0.05)
    no_device_errors()
    ref_default, _ = oracle_compact(wl, 0)
    assert_close(a, ref_default, "default scale")
    ref, _ = oracle_compact(wl, 0, scale=0.05)
    assert_close(c, ref, "explicit scale")


def test_strided_query_rows():
    wl = W.draw(tiny_spec(seed=9, head_dim=64, num_q_heads=8, num_kv_heads=2, block_size=16, num_blocks=200,
                          num_seqs=10, ctx_lo=1, ctx_hi=250))
    st = W.DeviceState(wl, DEV)
    run_store(st, 0)
    s = st.steps[0]
    q = s["q"]
    big = torch.zeros((wl.B, wl.Hq + 4, wl.D), dtype=torch.bfloat16, device=DEV)
    big[:, 2:2 + wl.Hq] = q
    qv = big[:, 2:2 + wl.Hq]
    out = ops.paged_decode_attention(qv, st.k_cache, st.v_cache, s["block_tables"], s["context_lens"])
    no_device_errors()
    ref, _ = oracle_compact(wl, 0)
    assert_close(out, ref, "strided q")


def test_decode_host_validation():
    l = ops.lib()
    dummy = torch.zeros(1024, dtype=torch.bfloat16, device=DEV)
    ptr = dummy.data_ptr()
    i32 = torch.zeros(16, dtype=torch.int32, device=DEV)
    ws = torch.zeros(1 << 20, dtype=torch.uint8, device=DEV)
    args = dict(out=ptr, q=ptr, qs=0, k=ptr, v=ptr, bt=i32.data_ptr(), mb=4, cl=i32.data_ptr(), B=2, Hq=8, Hkv=2,
                D=128, NB=4, BS=16, scale=0.0, ws=ws.data_ptr(), wsb=ws.numel())

    def call(**kw):
        a = dict(args)
        a.update(kw)
        return l.npv_paged_decode_attention(a["out"], a["q"], a["qs"], a["k"], a["v"], a["bt"], a["mb"], a["cl"],
                                            a["B"], a["Hq"], a["Hkv"], a["D"], a["NB"], a["BS"], a["scale"],
                                            a["ws"], a["wsb"], None)

    assert call(D=96) == 2
    assert call(Hq=6, Hkv=4) == 1
    assert call(Hq=24, Hkv=2) == 2  # g = 12
    assert call(BS=24) == 2
    assert call(wsb=16) == 3
    assert call(ws=ws.data_ptr() + 16) == 3
    assert call(q=ptr + 2) == 1
    assert call(B=0) == 0
    no_device_errors()
