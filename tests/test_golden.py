"""The oracle on the pages' own worked example (CPU).

tests/golden/xray_gqa_example.txt holds the shapes, the GQA ratio and the scale that
the "nano-vllm" README prints in its X-Ray walk-through (Layer 1, steps 1-2).  The
oracle, called with its default scale on exactly those shapes, must agree with a
library routine (torch's scaled_dot_product_attention in float64, given the
printed scale and grouping consecutive query heads per KV head) to rounding.
"""

import math
import os

import numpy as np

from cases import oracle_post_store, tiny_spec
from oracle import oracle as O
from paged_kv_cache_bf16_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "xray_gqa_example.txt")


def fixture():
    vals = {}
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        key, *rest = line.split()
        vals[key] = [float(x) if "." in x else int(x) for x in rest]
    return {k: (v[0] if len(v) == 1 else v) for k, v in vals.items()}


def test_printed_relations_hold():
    f = fixture()
    assert f["num_q_heads"] // f["num_kv_heads"] == f["q_heads_per_kv_head"]
    assert f["num_q_heads"] % f["num_kv_heads"] == 0
    assert abs(f["scale"] - 1.0 / math.sqrt(f["head_dim"])) < 1e-16
    assert f["scores_shape"] == [1, f["num_q_heads"], f["seq_len"], f["seq_len"]]


def test_oracle_on_the_printed_shapes_matches_library_attention():
    import torch
    import torch.nn.functional as F

    f = fixture()
    n, hq, hkv, d = f["seq_len"], f["num_q_heads"], f["num_kv_heads"], f["head_dim"]
    # the 5-token prompt as one prefill chunk with no prior context
    wl = W.draw(tiny_spec(name="xray", seed=1201, num_seqs=1, num_q_heads=hq, num_kv_heads=hkv, head_dim=d,
                          block_size=16, num_blocks=4, prefill_seqs=1, prefill_len=n, prior_lo=0, prior_hi=0))
    kp, vp = oracle_post_store(wl)
    out = O.paged_attention(wl.q(), kp, vp, wl.block_tables(), wl.context_lens(), wl.cu_seqlens_q())  # default scale
    assert out.shape == (n, hq, d)
    blocks = wl.block_tables()[0, :1]
    K = O.bf16_to_f64(kp[blocks].reshape(-1, hkv, d)[:n])
    V = O.bf16_to_f64(vp[blocks].reshape(-1, hkv, d)[:n])
    Q = O.bf16_to_f64(wl.q())
    scores_shape = (1, hq, n, n)
    assert list(scores_shape) == f["scores_shape"]
    ref = F.scaled_dot_product_attention(torch.from_numpy(Q).permute(1, 0, 2)[None],
                                         torch.from_numpy(K).permute(1, 0, 2)[None],
                                         torch.from_numpy(V).permute(1, 0, 2)[None],
                                         is_causal=True, scale=f["scale"], enable_gqa=True)
    ref = ref[0].permute(1, 0, 2).numpy()
    assert np.max(np.abs(out - ref)) < 1e-12
    # the 4:1 sharing: query heads 4k .. 4k+3 read KV head k, so swapping two KV heads'
    # contents permutes exactly those groups of outputs
    kp2, vp2 = kp.copy(), vp.copy()
    kp2[..., [0, 1], :] = kp[..., [1, 0], :]
    vp2[..., [0, 1], :] = vp[..., [1, 0], :]
    out2 = O.paged_attention(wl.q(), kp2, vp2, wl.block_tables(), wl.context_lens(), wl.cu_seqlens_q())
    g = f["q_heads_per_kv_head"]
    assert not np.allclose(out2[:, :g], out[:, :g])
    assert np.array_equal(out2[:, 2 * g:], out[:, 2 * g:])
