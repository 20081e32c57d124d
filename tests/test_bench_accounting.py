"""bench.py's algorithmic byte and FLOP counts, checked against closed forms (CPU)."""

import os
import sys

import numpy as np

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402
from paged_kv_cache_bf16_b200 import workloads as W  # noqa: E402


def test_unique_bytes_count_each_shared_block_once():
    wl = W.workload("llama8b_prefix_decode")
    s = wl.spec
    seqs = np.arange(wl.B)
    logical, unique = bench.kv_tokens(wl, 0, seqs)
    assert logical == int(wl.context_lens(0).sum())
    # every sequence reads all of its shared blocks in full (contexts exceed them), so each
    # group of `share_group` readers is counted once instead of share_group times
    groups = s.num_seqs // s.share_group
    extra = groups * (s.share_group - 1) * s.shared_blocks * s.block_size
    assert logical - unique == extra
    store, attn_u = bench.step_bytes(wl, 0)
    _, attn_l = bench.step_bytes(wl, 0, logical=True)
    row = 2 * s.num_kv_heads * s.head_dim * 2
    assert attn_l - attn_u == extra * row


def test_private_blocks_logical_equals_unique():
    wl = W.workload("qwen3_decode")
    for step in (0, 63):
        logical, unique = bench.kv_tokens(wl, step, np.arange(wl.B))
        assert logical == unique == int(wl.context_lens(step).sum())
    store, attn = bench.step_bytes(wl, 0)
    # store: read + write of one K and one V row per sequence
    assert store == 2 * wl.B * wl.Hkv * wl.D * 2 * 2


def test_prefill_flops_closed_form():
    # one sequence, n rows over a prior p: sum_i (p + i + 1) visible keys per row
    spec = W.Spec(name="f", seed=1, num_seqs=1, num_q_heads=4, num_kv_heads=2, head_dim=64, block_size=16,
                  num_blocks=64, prefill_seqs=1, prefill_len=50, prior_lo=100, prior_hi=100)
    wl = W.draw(spec)
    n, p = 50, 100
    pairs = n * p + n * (n + 1) // 2
    assert bench.prefill_flops(wl) == 4 * 64 * 4 * pairs
