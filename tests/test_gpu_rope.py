"""RoPE on q and k fused with the store of k and v (GPU), against the fp64 oracle.

The kernel turns each pair (x[i], x[i + D/2]) by p * base^(-2i/D) with the angle,
cos and sin in double precision, the rotation in fp32, and one rounding to bf16.
Bar for every rotated element: |gpu - exact| <= half a bf16 spacing at the exact
value (the one rounding) + EPS * r, r the pair's length |(x[i], x[i + D/2])| (the
fp32 rotation: cos and sin rounded to fp32, one product and one fused
multiply-add, each off by at most 2^-24 of a term bounded by r; EPS = 1e-6 is
about four times their sum).  Values are copied bit for bit; no other cache
byte changes.  Whole steps (RoPE + store, then decode or prefill attention) meet
the attention tolerance against the oracle's rotate-round-store-attend.
"""

import numpy as np
import pytest
import torch

from cases import tiny_spec
from gpu_common import DEV, assert_close, no_device_errors
from oracle import oracle as O
from paged_kv_cache_bf16_b200 import ops
from paged_kv_cache_bf16_b200 import workloads as W

pytestmark = pytest.mark.gpu

EPS = 1e-6


def _bits(rng, shape):
    return W.f32_to_bf16_bits(rng.standard_normal(shape).astype(np.float32))


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def _as_bf16(bits):
    return _dev(bits.view(np.int16)).view(torch.bfloat16)


def _host_bits(t):
    return t.detach().cpu().view(torch.int16).numpy().view(np.uint16)


def _check_rotated(got_bits, x_bits, exact, what):
    """got_bits, x_bits: [..., D] bf16 bits; exact: fp64 rotation of x."""
    got = O.bf16_to_f64(got_bits)
    x = O.bf16_to_f64(x_bits)
    h = x.shape[-1] // 2
    r_half = np.sqrt(x[..., :h] ** 2 + x[..., h:] ** 2)
    r = np.concatenate([r_half, r_half], axis=-1)
    mag = np.maximum(np.abs(exact) + EPS * r, 2.0 ** -126)
    spacing = np.exp2(np.floor(np.log2(mag)) - 7)
    err = np.abs(got - exact)
    tol = 0.5 * spacing + EPS * r
    bad = err > tol
    assert not bad.any(), f"{what}: {int(bad.sum())} elements off, worst excess {float((err - tol).max()):.3e}"
    # nearly every element is the correctly rounded bf16 of the exact value
    same = np.mean(got_bits == O.to_bf16(exact))
    assert same >= 0.99, f"{what}: only {same:.4f} equal the nearest bf16"


CASES = [
    # (D, Hq, Hkv, T, base)
    (128, 16, 8, 301, 1.0e6),
    (64, 8, 2, 77, 1.0e4),
    (128, 32, 8, 5, 1.0e6),
    (128, 8, 8, 1, 5.0e5),
    (256, 4, 1, 9, 1.0e4),
    (16, 2, 1, 13, 1.0e6),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "D%d_q%d_kv%d_T%d" % c[:4])
def test_rope_store_rows(case):
    D, Hq, Hkv, T, base = case
    rng = np.random.default_rng(7000 + D + T)
    BS = 16
    NB = T // BS + 3
    q = _bits(rng, (T, Hq, D))
    key = _bits(rng, (T, Hkv, D))
    val = _bits(rng, (T, Hkv, D))
    pos = rng.integers(0, 1 << 17, T).astype(np.int32)
    pos[: min(T, 3)] = [0, 131071, 1][: min(T, 3)]
    slots = rng.permutation(NB * BS)[:T].astype(np.int32)
    slots[3::7] = -1  # padding rows store nothing
    kc0 = _bits(rng, (NB, BS, Hkv, D))
    vc0 = _bits(rng, (NB, BS, Hkv, D))

    qg, kc, vc = _as_bf16(q), _as_bf16(kc0), _as_bf16(vc0)
    ops.rope_store_kvcache(qg, _as_bf16(key), _as_bf16(val), _dev(pos), kc, vc, _dev(slots), base)
    no_device_errors()

    _check_rotated(_host_bits(qg), q, O.rope(q, pos, base), "q")
    kr = O.rope(key, pos, base)
    k_after = _host_bits(kc).reshape(NB * BS, Hkv, D)
    v_after = _host_bits(vc).reshape(NB * BS, Hkv, D)
    live = slots >= 0
    _check_rotated(k_after[slots[live]], key[live], kr[live], "k in cache")
    assert np.array_equal(v_after[slots[live]], val[live])
    untouched = np.ones(NB * BS, dtype=bool)
    untouched[slots[live]] = False
    assert np.array_equal(k_after[untouched], kc0.reshape(NB * BS, Hkv, D)[untouched])
    assert np.array_equal(v_after[untouched], vc0.reshape(NB * BS, Hkv, D)[untouched])


def test_rope_store_key_only_and_bad_slot():
    """q = None rotates and stores k only; a slot past the cache sets NPV_DEVERR_SLOT
    and stores nothing for that token, while the others are stored."""
    rng = np.random.default_rng(7100)
    D, Hkv, T, NB, BS = 128, 4, 12, 2, 16
    key = _bits(rng, (T, Hkv, D))
    val = _bits(rng, (T, Hkv, D))
    pos = rng.integers(0, 5000, T).astype(np.int32)
    slots = rng.permutation(NB * BS)[:T].astype(np.int32)
    slots[5] = NB * BS + 3
    kc0 = _bits(rng, (NB, BS, Hkv, D))
    vc0 = _bits(rng, (NB, BS, Hkv, D))
    kc, vc = _as_bf16(kc0), _as_bf16(vc0)
    ops.rope_store_kvcache(None, _as_bf16(key), _as_bf16(val), _dev(pos), kc, vc, _dev(slots), 1.0e6)
    with pytest.raises(ops.NpvError) as ei:
        ops.check_device_errors()
    assert ei.value.bits == 0x1
    ok = np.arange(T) != 5
    k_after = _host_bits(kc).reshape(NB * BS, Hkv, D)
    _check_rotated(k_after[slots[ok]], key[ok], O.rope(key, pos, 1.0e6)[ok], "k")
    assert np.array_equal(_host_bits(vc).reshape(NB * BS, Hkv, D)[slots[ok]], val[ok])
    no_device_errors()


def _oracle_rope_step(wl, base):
    """The oracle's step: rotate q and k (fp64, rounded to bf16), store k and v, attend."""
    _, pos = wl.token_positions(0)
    kp, vp = wl.host_pool()
    k, v = wl.new_kv(0)
    qbits, _, _ = O.rope_store_kvcache(wl.q(0), k, v, pos.astype(np.int32), kp, vp, wl.slot_mapping(0), base)
    return O.paged_attention(qbits, kp, vp, wl.block_tables(0), wl.context_lens(0), wl.cu_seqlens_q())


@pytest.mark.parametrize("hq,hkv", [(16, 8), (32, 8)])
def test_rope_decode_step(hq, hkv):
    """A decode step with RoPE: rope + store, then decode attention with the rotated q."""
    wl = W.draw(tiny_spec(name="rope_decode", seed=7200 + hq, num_seqs=24, num_q_heads=hq, num_kv_heads=hkv,
                          head_dim=128, block_size=16, num_blocks=1400, ctx_lo=1, ctx_hi=900))
    st = W.DeviceState(wl, DEV)
    s = st.steps[0]
    _, pos = wl.token_positions(0)
    q = s["q"].clone()
    ops.rope_store_kvcache(q, s["key"], s["value"], _dev(pos.astype(np.int32)), st.k_cache, st.v_cache,
                           s["slot_mapping"], 1.0e6)
    out = ops.paged_decode_attention(q, st.k_cache, st.v_cache, s["block_tables"], s["context_lens"])
    no_device_errors()
    assert_close(out, _oracle_rope_step(wl, 1.0e6), "rope decode step")


def test_rope_chunked_prefill_step():
    """A mixed batch with RoPE: prefill chunks over cached context and decode rows,
    each new row rotated at its own position, then the varlen causal attention."""
    wl = W.draw(tiny_spec(name="rope_prefill", seed=7300, num_seqs=10, num_q_heads=16, num_kv_heads=8,
                          head_dim=128, block_size=16, num_blocks=600, ctx_lo=1, ctx_hi=400, prefill_seqs=4,
                          prefill_len=150, prior_lo=0, prior_hi=500))
    st = W.DeviceState(wl, DEV)
    s = st.steps[0]
    _, pos = wl.token_positions(0)
    q = s["q"].clone()
    ops.rope_store_kvcache(q, s["key"], s["value"], _dev(pos.astype(np.int32)), st.k_cache, st.v_cache,
                           s["slot_mapping"], 1.0e4)
    out = ops.paged_prefill_attention(q, st.k_cache, st.v_cache, s["cu_seqlens_q"], s["max_seqlen_q"],
                                      s["block_tables"], s["context_lens"])
    no_device_errors()
    assert_close(out, _oracle_rope_step(wl, 1.0e4), "rope prefill step")
