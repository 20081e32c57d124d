"""The seeded input generator: determinism, rounding, distributions, metadata validity (CPU)."""

import numpy as np
import pytest
import torch

from paged_kv_cache_bf16_b200 import workloads as W


def test_splitmix64_reference_values():
    # SplitMix64 seeded with 0: first outputs as published with the generator
    g = W.SplitMix64(0)
    assert [g.next_u64() for _ in range(3)] == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.normal(size=20000).astype(np.float32) * 3,
                        np.array([1.00390625, 1.01171875, -2.00781250, 65504.0, 1e-30, -0.0], np.float32)])
    ours = W.f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


def test_normal_stream_deterministic_and_random_access():
    k = W.stream_key(7, W.TAG_Q, 0)
    a = W.normal_bf16(k, 0, 10000)
    assert np.array_equal(a, W.normal_bf16(k, 0, 10000))
    assert np.array_equal(a[1234:5678], W.normal_bf16(k, 1234, 5678 - 1234))
    big = W.normal_bf16(k, 0, (1 << 22) + 999)  # crosses the threaded chunking
    assert np.array_equal(big[:10000], a)
    assert np.array_equal(big[(1 << 22) - 5:(1 << 22) + 5], W.normal_bf16(k, (1 << 22) - 5, 10))


@pytest.mark.parametrize("sigma", [1.0, 0.5])
def test_normal_moments(sigma):
    x = W.bf16_bits_to_f32(W.normal_bf16(W.stream_key(3, 99), 0, 400000, sigma)).astype(np.float64)
    assert abs(x.mean()) < 0.01 * sigma
    assert abs(x.std() - sigma) < 0.01 * sigma
    assert abs((np.abs(x) < sigma).mean() - 0.6827) < 0.005


@pytest.mark.parametrize("name", sorted(W.SPECS))
def test_named_workload_metadata(name):
    wl = W.workload(name)
    s = wl.spec
    L = wl.context_lens(0)
    assert L.shape == (s.num_seqs,) and (L >= wl.query_lens).all()
    if s.prefill_seqs:
        pre = wl.query_lens > 1
        assert pre.sum() == s.prefill_seqs and (wl.query_lens[pre] == s.prefill_len).all()
        prior = L[pre] - s.prefill_len
        assert prior.min() >= s.prior_lo and prior.max() <= s.prior_hi
        if (~pre).any():
            assert L[~pre].min() >= s.ctx_lo and L[~pre].max() <= s.ctx_hi
    else:
        assert L.min() >= s.ctx_lo and L.max() <= s.ctx_hi
    for step in (0, s.num_steps - 1):
        bt = wl.block_tables(step)
        Ls = wl.context_lens(step)
        live = []
        for b in range(s.num_seqs):
            nb = -(-int(Ls[b]) // s.block_size)
            assert (bt[b, :nb] >= 0).all() and (bt[b, :nb] < s.num_blocks).all()
            assert (bt[b, nb:] == -1).all()
            live.extend(bt[b, s.shared_blocks if s.share_group else 0:nb].tolist())
        assert len(live) == len(set(live)), "private blocks must not repeat"
        slots = wl.slot_mapping(step)
        assert len(np.unique(slots)) == len(slots)
        assert slots.min() >= 0 and slots.max() < s.num_blocks * s.block_size
    if s.share_group:
        bt = wl.block_tables(0)
        for g0 in range(0, s.num_seqs, s.share_group):
            grp = bt[g0:g0 + s.share_group, :s.shared_blocks]
            assert (grp == grp[0]).all()
        # new tokens never land in a shared block
        shared = set(bt[:, :s.shared_blocks].ravel().tolist())
        assert not (set((wl.slot_mapping(0) // s.block_size).tolist()) & shared)


def test_prior_fill_covers_cached_prefix_only():
    wl = W.draw(W.Spec(name="t", seed=9, num_seqs=3, num_q_heads=2, num_kv_heads=1, head_dim=8, block_size=4,
                       num_blocks=20, ctx_lo=1, ctx_hi=11))
    kp, vp = wl.host_pool()
    flat = kp.reshape(-1, 8)
    nan_rows = (flat == W.BF16_NAN).all(axis=1)
    bt = wl.block_tables(0)
    expect_nan = np.ones(20 * 4, dtype=bool)
    for b in range(3):
        for j in range(wl.prior_len(b)):
            expect_nan[bt[b, j // 4] * 4 + j % 4] = False
    assert np.array_equal(nan_rows, expect_nan)


def test_qwen3_decode_steps_pop_blocks_in_order():
    wl = W.workload("qwen3_decode")
    L0, L63 = wl.context_lens(0), wl.context_lens(63)
    assert (L63 - L0 == 63).all()
    bt0, bt63 = wl.block_tables(0), wl.block_tables(63)
    grew = -(-L63 // 256) > -(-L0 // 256)
    assert grew.any()
    assert ((bt63[:, :bt0.shape[1]] == bt0) | (bt0 == -1)).all()
