"""Pins of the fp64 oracle to facts fixed outside itself.

Each check takes an oracle build (`lib`, a ctypes handle) and raises
AssertionError (or OracleError) when the pin fails, so the same checks run
against the real oracle (tests/test_oracle_pins.py) and against copies with a
planted mistake (tests/test_oracle_mutations.py), which at least one check must
catch.  What pins what:

  store layout   literal tiny example; gather-after-store round trip; untouched
                 slots unchanged
  scale          two-token closed form sigma(scale * <q, k1 - k0>) at D = 8, 64, 128
  normalisation  equal keys give the mean of V; one-token context returns V
  mask / gather  pure-Python brute force (tests/bruteforce.py, written separately)
  GQA            equals the MHA form with each KV head repeated g times
  library        torch scaled_dot_product_attention in float64 (enable_gqa)
  paging         contiguous relabelling and random relabelling of blocks
  chunking       one chunk equals two successive chunks; a prefill row equals
                 decode over the truncated context
  prefix sharing shared physical blocks equal private copies
  rope           unit vectors at whole-radian angles (tests/golden/rope_worked_example.txt);
                 the complex-product form with numpy's complex exponential; the
                 relative-position identity and pair lengths; position 0 is the identity
  bf16 rounding  the input generator's fp32 bit-level rounding; hand-worked ties and limits
"""

from __future__ import annotations

import math
import os

import numpy as np

from cases import oracle_attention, oracle_post_store, tiny_spec
from oracle import oracle as O
from paged_kv_cache_bf16_b200 import workloads as W

import bruteforce


def _bits(x) -> np.ndarray:
    return W.f32_to_bf16_bits(np.asarray(x, dtype=np.float32))


def _f64(bits) -> np.ndarray:
    return O.bf16_to_f64(bits)


# ---------------------------------------------------------------- store ----

def check_store_literal(lib) -> None:
    """NB=3, BS=2, Hkv=1, D=2: slot 5 is block 2 offset 1, slot 0 is block 0 offset 0."""
    kp = (np.arange(12, dtype=np.uint16) + 1000).reshape(3, 2, 1, 2)
    vp = (np.arange(12, dtype=np.uint16) + 2000).reshape(3, 2, 1, 2)
    key = np.array([[[1, 2]], [[3, 4]], [[5, 6]]], dtype=np.uint16)
    val = np.array([[[7, 8]], [[9, 10]], [[11, 12]]], dtype=np.uint16)
    O.store_kvcache(key, val, kp, vp, np.array([5, 0, -1], dtype=np.int32), _lib=lib)
    ek = np.array([[[[3, 4]], [[1002, 1003]]], [[[1004, 1005]], [[1006, 1007]]],
                   [[[1008, 1009]], [[1, 2]]]], dtype=np.uint16)
    ev = np.array([[[[9, 10]], [[2002, 2003]]], [[[2004, 2005]], [[2006, 2007]]],
                   [[[2008, 2009]], [[7, 8]]]], dtype=np.uint16)
    assert np.array_equal(kp, ek), kp
    assert np.array_equal(vp, ev), vp


def check_store_roundtrip(lib) -> None:
    wl = W.draw(tiny_spec(seed=202, num_seqs=6, prefill_seqs=2, prefill_len=5, prior_lo=0, prior_hi=9))
    kp, vp = wl.host_pool()
    k0, v0 = kp.copy(), vp.copy()
    key, val = wl.new_kv(0)
    slots = wl.slot_mapping(0)
    O.store_kvcache(key, val, kp, vp, slots, _lib=lib)
    flat_k = kp.reshape(-1, wl.Hkv, wl.D)
    flat_v = vp.reshape(-1, wl.Hkv, wl.D)
    assert np.array_equal(flat_k[slots], key)
    assert np.array_equal(flat_v[slots], val)
    untouched = np.ones(flat_k.shape[0], dtype=bool)
    untouched[slots] = False
    assert np.array_equal(flat_k[untouched], k0.reshape(-1, wl.Hkv, wl.D)[untouched])
    assert np.array_equal(flat_v[untouched], v0.reshape(-1, wl.Hkv, wl.D)[untouched])


def check_store_rejects_out_of_range(lib) -> None:
    kp = np.zeros((2, 2, 1, 2), dtype=np.uint16)
    vp = np.zeros_like(kp)
    key = np.ones((1, 1, 2), dtype=np.uint16)
    try:
        O.store_kvcache(key, key, kp, vp, np.array([4], dtype=np.int32), _lib=lib)
    except O.OracleError:
        return
    raise AssertionError("slot == num_blocks * block_size was accepted")


# ------------------------------------------------------- closed forms ----

def _single_seq(keys_f32, vals_f32, q_f32, block_size=16):
    """One sequence, Hq = Hkv = 1, keys/values [L, D] laid in a 1-seq pool."""
    keys = _bits(keys_f32)
    vals = _bits(vals_f32)
    L, D = keys.shape
    nblk = -(-L // block_size)
    kp = np.full((nblk + 2, block_size, 1, D), W.BF16_NAN, dtype=np.uint16)
    vp = kp.copy()
    # physical blocks in reverse order, to keep the paging in play
    bt = np.array([[nblk + 1 - i for i in range(nblk)]], dtype=np.int32)
    for j in range(L):
        kp[bt[0, j // block_size], j % block_size, 0] = keys[j]
        vp[bt[0, j // block_size], j % block_size, 0] = vals[j]
    q = _bits(q_f32).reshape(1, 1, D)
    return q, kp, vp, bt, np.array([L], dtype=np.int32), keys, vals


def check_one_token_returns_v(lib) -> None:
    rng = np.random.default_rng(5)
    for D in (8, 64, 128):
        q, kp, vp, bt, L, keys, vals = _single_seq(rng.normal(size=(1, D)), rng.normal(size=(1, D)),
                                                   rng.normal(size=D) * 3)
        out = O.decode_attention(q, kp, vp, bt, L, _lib=lib)
        assert np.array_equal(out[0, 0], _f64(vals[0])), (out[0, 0], _f64(vals[0]))
    # many query heads on one KV head, several sequences of length 1
    wl = W.draw(tiny_spec(seed=303, num_q_heads=6, num_kv_heads=1, ctx_lo=1, ctx_hi=1, num_seqs=5))
    kp, vp = oracle_post_store(wl, lib=lib)
    out = oracle_attention(wl, kp, vp, lib=lib)
    _, newv = wl.new_kv(0)
    for b in range(wl.B):
        for h in range(wl.Hq):
            assert np.array_equal(out[b, h], _f64(newv[b, 0]))


def check_two_token_closed_form(lib) -> None:
    rng = np.random.default_rng(7)
    for D in (8, 64, 128):
        for trial in range(4):
            q, kp, vp, bt, L, keys, vals = _single_seq(rng.normal(size=(2, D)), rng.normal(size=(2, D)),
                                                       rng.normal(size=D) * (1 + trial))
            qf, k0, k1 = _f64(q[0, 0]), _f64(keys[0]), _f64(keys[1])
            delta = math.fsum(qf * (k1 - k0)) / math.sqrt(D)
            sig = 1.0 / (1.0 + math.exp(-delta))
            expect = sig * _f64(vals[1]) + (1.0 - sig) * _f64(vals[0])
            out = O.decode_attention(q, kp, vp, bt, L, _lib=lib)
            assert np.max(np.abs(out[0, 0] - expect)) < 1e-12, (D, delta, out[0, 0][:4], expect[:4])


def check_explicit_scale(lib) -> None:
    rng = np.random.default_rng(9)
    D = 16
    q, kp, vp, bt, L, keys, vals = _single_seq(rng.normal(size=(2, D)), rng.normal(size=(2, D)), rng.normal(size=D))
    s = 0.37
    qf, k0, k1 = _f64(q[0, 0]), _f64(keys[0]), _f64(keys[1])
    sig = 1.0 / (1.0 + math.exp(-s * math.fsum(qf * (k1 - k0))))
    expect = sig * _f64(vals[1]) + (1.0 - sig) * _f64(vals[0])
    out = O.decode_attention(q, kp, vp, bt, L, scale=s, _lib=lib)
    assert np.max(np.abs(out[0, 0] - expect)) < 1e-12


def check_equal_keys_mean(lib) -> None:
    rng = np.random.default_rng(11)
    D, L = 32, 21
    key = rng.normal(size=D)
    q, kp, vp, bt, Ls, keys, vals = _single_seq(np.tile(key, (L, 1)), rng.normal(size=(L, D)), rng.normal(size=D) * 4,
                                                block_size=8)
    out = O.decode_attention(q, kp, vp, bt, Ls, _lib=lib)
    expect = np.array([math.fsum(_f64(vals[:, d])) / L for d in range(D)])
    assert np.max(np.abs(out[0, 0] - expect)) < 1e-13


# -------------------------------------------------------- references ----

def _mixed_tiny(seed: int = 404) -> W.Workload:
    return W.draw(tiny_spec(seed=seed, num_seqs=5, prefill_seqs=2, prefill_len=5, prior_lo=0, prior_hi=9,
                            ctx_lo=1, ctx_hi=14))


def check_brute_force(lib) -> None:
    for seed in (404, 405):
        wl = _mixed_tiny(seed)
        kp, vp = oracle_post_store(wl, lib=lib)
        out = oracle_attention(wl, kp, vp, lib=lib)
        ref = np.array(bruteforce.attention(wl.q(), kp, vp, wl.block_tables(), wl.context_lens(), wl.cu_seqlens_q()))
        assert np.max(np.abs(out - ref)) < 1e-12, np.max(np.abs(out - ref))


def check_torch_sdpa(lib) -> None:
    import torch
    import torch.nn.functional as F

    # decode batch and a prior-free causal prefill, against the library routine
    wl = W.draw(tiny_spec(seed=505, num_seqs=4, num_q_heads=8, num_kv_heads=2, head_dim=16, ctx_lo=3, ctx_hi=30))
    for prefill in (False, True):
        if prefill:
            wl = W.draw(tiny_spec(seed=506, num_seqs=3, num_q_heads=8, num_kv_heads=2, head_dim=16,
                                  prefill_seqs=3, prefill_len=7, prior_lo=0, prior_hi=0))
        kp, vp = oracle_post_store(wl, lib=lib)
        out = oracle_attention(wl, kp, vp, lib=lib)
        q = _f64(wl.q())
        cu = wl.cu_seqlens_q()
        L = wl.context_lens()
        bt = wl.block_tables()
        for b in range(wl.B):
            blocks = bt[b, : -(-int(L[b]) // wl.BS)]
            K = _f64(kp[blocks].reshape(-1, wl.Hkv, wl.D)[: L[b]])  # [L, Hkv, D]
            V = _f64(vp[blocks].reshape(-1, wl.Hkv, wl.D)[: L[b]])
            Q = q[cu[b]:cu[b + 1]]  # [n, Hq, D]
            r = F.scaled_dot_product_attention(torch.from_numpy(Q).permute(1, 0, 2)[None],
                                               torch.from_numpy(K).permute(1, 0, 2)[None],
                                               torch.from_numpy(V).permute(1, 0, 2)[None],
                                               is_causal=prefill, enable_gqa=True)
            r = r[0].permute(1, 0, 2).numpy()
            assert np.max(np.abs(out[cu[b]:cu[b + 1]] - r)) < 1e-12, (b, np.max(np.abs(out[cu[b]:cu[b + 1]] - r)))


# ------------------------------------------------------------ invariants ----

def check_paging_contiguous(lib) -> None:
    """Shuffled block tables give exactly what consecutive blocks give."""
    wl = _mixed_tiny(606)
    kp, vp = oracle_post_store(wl, lib=lib)
    out = oracle_attention(wl, kp, vp, lib=lib)
    bt = wl.block_tables()
    L = wl.context_lens()
    kc = np.full_like(kp, W.BF16_NAN)
    vc = np.full_like(vp, W.BF16_NAN)
    bt2 = np.full_like(bt, -1)
    nxt = 0
    for b in range(wl.B):
        for i in range(-(-int(L[b]) // wl.BS)):
            kc[nxt], vc[nxt] = kp[bt[b, i]], vp[bt[b, i]]
            bt2[b, i] = nxt
            nxt += 1
    out2 = O.paged_attention(wl.q(), kc, vc, bt2, L, wl.cu_seqlens_q(), _lib=lib)
    assert np.array_equal(out, out2)


def check_relabel(lib) -> None:
    wl = _mixed_tiny(707)
    kp, vp = oracle_post_store(wl, lib=lib)
    out = oracle_attention(wl, kp, vp, lib=lib)
    perm = np.random.default_rng(1).permutation(wl.NB)
    k2 = np.empty_like(kp)
    v2 = np.empty_like(vp)
    k2[perm] = kp
    v2[perm] = vp
    bt = wl.block_tables()
    bt2 = np.where(bt >= 0, perm[np.maximum(bt, 0)], -1).astype(np.int32)
    out2 = O.paged_attention(wl.q(), k2, v2, bt2, wl.context_lens(), wl.cu_seqlens_q(), _lib=lib)
    assert np.array_equal(out, out2)


def check_gqa_repeat(lib) -> None:
    """Hkv KV heads shared by g query heads == MHA with each KV head repeated g times."""
    wl = W.draw(tiny_spec(seed=808, num_q_heads=8, num_kv_heads=2, num_seqs=4, prefill_seqs=1, prefill_len=4,
                          prior_lo=1, prior_hi=6))
    kp, vp = oracle_post_store(wl, lib=lib)
    out = oracle_attention(wl, kp, vp, lib=lib)
    g = wl.Hq // wl.Hkv
    kr = np.ascontiguousarray(np.repeat(kp, g, axis=2))
    vr = np.ascontiguousarray(np.repeat(vp, g, axis=2))
    out2 = O.paged_attention(wl.q(), kr, vr, wl.block_tables(), wl.context_lens(), wl.cu_seqlens_q(), _lib=lib)
    assert np.array_equal(out, out2)


def _one_prefill_seq(seed: int, prior: int, n: int, lib):
    wl = W.draw(tiny_spec(seed=seed, num_seqs=1, prefill_seqs=1, prefill_len=n, prior_lo=prior, prior_hi=prior))
    kp, vp = oracle_post_store(wl, lib=lib)
    return wl, kp, vp


def check_chunk_split(lib) -> None:
    """A 12-row chunk equals an 8-row chunk followed by a 4-row chunk."""
    prior, n, n1 = 5, 12, 8
    wl, kp, vp = _one_prefill_seq(909, prior, n, lib)
    q = wl.q()
    bt = wl.block_tables()
    out = O.paged_attention(q, kp, vp, bt, np.array([prior + n], np.int32), np.array([0, n], np.int32), _lib=lib)
    a = O.paged_attention(q[:n1], kp, vp, bt, np.array([prior + n1], np.int32), np.array([0, n1], np.int32), _lib=lib)
    b = O.paged_attention(q[n1:], kp, vp, bt, np.array([prior + n], np.int32), np.array([0, n - n1], np.int32),
                          _lib=lib)
    assert np.array_equal(out, np.concatenate([a, b]))


def check_prefill_row_is_decode(lib) -> None:
    prior, n = 6, 7
    wl, kp, vp = _one_prefill_seq(910, prior, n, lib)
    q = wl.q()
    bt = wl.block_tables()
    out = O.paged_attention(q, kp, vp, bt, np.array([prior + n], np.int32), np.array([0, n], np.int32), _lib=lib)
    for i in range(n):
        d = O.decode_attention(q[i:i + 1], kp, vp, bt, np.array([prior + i + 1], np.int32), _lib=lib)
        assert np.array_equal(out[i], d[0]), i


def check_prefix_sharing(lib) -> None:
    wl = W.draw(tiny_spec(seed=911, num_seqs=6, share_group=3, shared_blocks=2, ctx_lo=9, ctx_hi=20, num_blocks=64))
    kp, vp = oracle_post_store(wl, lib=lib)
    out = oracle_attention(wl, kp, vp, lib=lib)
    bt = wl.block_tables()
    # give every sequence private copies of its shared blocks
    used = set(int(x) for x in bt.ravel() if x >= 0)
    free = [p for p in range(wl.NB) if p not in used]
    bt2 = bt.copy()
    k2, v2 = kp.copy(), vp.copy()
    for b in range(wl.B):
        for i in range(wl.spec.shared_blocks):
            p = free.pop()
            k2[p], v2[p] = kp[bt[b, i]], vp[bt[b, i]]
            bt2[b, i] = p
    assert len(set(bt[:, 0])) < wl.B  # sharing really happened
    out2 = O.paged_attention(wl.q(), k2, v2, bt2, wl.context_lens(), wl.cu_seqlens_q(), _lib=lib)
    assert np.array_equal(out, out2)


def check_nan_never_read(lib) -> None:
    wl = _mixed_tiny(912)
    kp, vp = oracle_post_store(wl, lib=lib)
    assert np.isnan(_f64(kp)).any()  # the pool is poisoned outside live tokens
    out = oracle_attention(wl, kp, vp, lib=lib)
    assert np.isfinite(out).all()


def check_invalid_inputs(lib) -> None:
    wl = _mixed_tiny(913)
    kp, vp = oracle_post_store(wl, lib=lib)
    q, cu, L = wl.q(), wl.cu_seqlens_q(), wl.context_lens()
    bad_bt = wl.block_tables()
    bad_bt[0, 0] = wl.NB
    bad_L = L.copy()
    bad_L[int(np.argmax(wl.query_lens))] = int(wl.query_lens.max()) - 1
    for bt, Ls in ((bad_bt, L), (wl.block_tables(), bad_L)):
        try:
            O.paged_attention(q, kp, vp, bt, Ls, cu, _lib=lib)
        except O.OracleError:
            continue
        raise AssertionError("invalid input accepted")


def check_threads_agree(lib) -> None:
    wl = _mixed_tiny(914)
    kp, vp = oracle_post_store(wl, lib=lib)
    a = oracle_attention(wl, kp, vp, lib=lib, threads=1)
    b = oracle_attention(wl, kp, vp, lib=lib, threads=7)
    assert np.array_equal(a, b)


# ------------------------------------------------------------------ rope ----

ROPE_GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "rope_worked_example.txt")


def rope_golden_rows():
    rows = []
    for line in open(ROPE_GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        f = line.split()
        D, base, pos, unit = int(f[0]), float(f[1]), int(f[2]), int(f[3])
        expect = np.array([float(v) for v in f[4:]])
        assert expect.shape == (D,)
        rows.append((D, base, pos, unit, expect))
    return rows


def check_rope_worked_example(lib) -> None:
    """Unit vectors at positions where p * theta_i is a whole number of radians."""
    rows = rope_golden_rows()
    assert len(rows) >= 10
    for D, base, pos, unit, expect in rows:
        x = np.zeros((1, 1, D), dtype=np.float32)
        x[0, 0, unit] = 1.0
        out = O.rope(_bits(x), np.array([pos], dtype=np.int32), base, _lib=lib)[0, 0]
        assert np.max(np.abs(out - expect)) < 1e-14, (D, base, pos, unit, out, expect)


def check_rope_position_zero(lib) -> None:
    rng = np.random.default_rng(31)
    x = _bits(rng.standard_normal((4, 3, 64)))
    out = O.rope(x, np.zeros(4, dtype=np.int32), 1.0e6, _lib=lib)
    assert np.array_equal(out, _f64(x))


def check_rope_complex_product(lib) -> None:
    """The rotation is the complex product z_i exp(j p theta_i), z_i = x_i + j x_{i+D/2}
    (numpy's complex exponential; theta_i = base^(-2i/D), RoFormer section 3.4)."""
    rng = np.random.default_rng(32)
    pos = np.array([0, 1, 7, 4095, 40959, 131071], dtype=np.int32)
    for D in (8, 64, 128):
        for base in (1.0e4, 1.0e6):
            x = _bits(rng.standard_normal((pos.size, 3, D)))
            f = _f64(x)
            h = D // 2
            theta = np.power(base, -np.arange(h, dtype=np.float64) * 2.0 / D)
            w = (f[..., :h] + 1j * f[..., h:]) * np.exp(1j * pos[:, None, None].astype(np.float64) * theta)
            expect = np.concatenate([w.real, w.imag], axis=-1)
            out = O.rope(x, pos, base, _lib=lib)
            assert np.max(np.abs(out - expect)) < 1e-9, (D, base, np.max(np.abs(out - expect)))


def check_rope_relative_position(lib) -> None:
    """<R(m) q, R(n) k> = <R(m - n) q, k> (the property RoPE is built for) and each
    pair keeps its length."""
    rng = np.random.default_rng(33)
    D = 64
    q = _bits(rng.standard_normal((1, 4, D)))
    k = _bits(rng.standard_normal((1, 4, D)))
    for m, n in ((5, 3), (1000, 17), (70000, 69999), (12, 40)):
        qm = O.rope(q, np.array([m], dtype=np.int32), 1.0e6, _lib=lib)
        kn = O.rope(k, np.array([n], dtype=np.int32), 1.0e6, _lib=lib)
        qd = O.rope(q, np.array([m - n], dtype=np.int32), 1.0e6, _lib=lib)
        lhs = np.sum(qm * kn, axis=-1)
        rhs = np.sum(qd * _f64(k), axis=-1)
        assert np.max(np.abs(lhs - rhs)) < 1e-9, (m, n, lhs, rhs)
        h = D // 2
        r_in = _f64(q)[..., :h] ** 2 + _f64(q)[..., h:] ** 2
        r_out = qm[..., :h] ** 2 + qm[..., h:] ** 2
        assert np.max(np.abs(r_in - r_out)) < 1e-12


def check_rope_strided_rows(lib) -> None:
    """Rows are read token_stride apart and heads D apart: a token's heads and tokens
    do not mix (each [head] slice equals a one-head call on that slice)."""
    rng = np.random.default_rng(34)
    x = _bits(rng.standard_normal((5, 3, 16)))
    pos = np.array([3, 0, 9, 2, 7], dtype=np.int32)
    out = O.rope(x, pos, 1.0e4, _lib=lib)
    for t in range(5):
        for h in range(3):
            one = O.rope(x[t:t + 1, h:h + 1], pos[t:t + 1], 1.0e4, _lib=lib)[0, 0]
            assert np.array_equal(out[t, h], one), (t, h)


def check_to_bf16(lib) -> None:
    """Nearest bf16, ties to even: agrees with the bit-level fp32 rounding of the input
    generator on fp32-exact values, and on hand-worked ties and limits."""
    rng = np.random.default_rng(35)
    v = (rng.standard_normal(4096) * np.exp2(rng.integers(-140, 120, 4096))).astype(np.float32)
    assert np.array_equal(O.to_bf16(v.astype(np.float64), _lib=lib), W.f32_to_bf16_bits(v))
    cases = {
        1.0: 0x3F80, 1.0 + 2.0 ** -8: 0x3F80, 1.0 + 3 * 2.0 ** -8: 0x3F82, 1.0 + 2.0 ** -8 + 2.0 ** -40: 0x3F81,
        -2.5: 0xC020, 2.0 ** -133: 0x0001, 2.0 ** -134: 0x0000, 3 * 2.0 ** -134: 0x0002,
        255.0 * 2.0 ** 120: 0x7F7F, 511.0 * 2.0 ** 119: 0x7F80, -1e39: 0xFF80, 0.0: 0x0000,
    }
    for val, bits in cases.items():
        got = int(O.to_bf16(np.array([val]), _lib=lib)[0])
        assert got == bits, (val, hex(got), hex(bits))


ALL_CHECKS = [
    check_store_literal, check_store_roundtrip, check_store_rejects_out_of_range,
    check_one_token_returns_v, check_two_token_closed_form, check_explicit_scale, check_equal_keys_mean,
    check_brute_force, check_torch_sdpa, check_paging_contiguous, check_relabel, check_gqa_repeat,
    check_chunk_split, check_prefill_row_is_decode, check_prefix_sharing, check_nan_never_read,
    check_invalid_inputs, check_threads_agree,
    check_rope_worked_example, check_rope_position_zero, check_rope_complex_product, check_rope_relative_position,
    check_rope_strided_rows, check_to_bf16,
]
