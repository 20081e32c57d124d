"""Short multi-row sequences (speculative-decode verification, short chunks) in a
prefill call, against the fp64 oracle (GPU).

Sequences with g * n_b <= 16 query rows per KV head run on the split-KV decode
kernel's warp-level MMA tiles (one 8-column tile when the call's max_seqlen_q
hint says g * n_b <= 8, two otherwise); longer ones on the tcgen05 kernel.  Each
call here mixes decode rows, short multi-row sequences and longer chunks, with
contexts long enough that most (sequence, KV head) units are cut across CTAs
and merged.  Every row is checked; a row i of a sequence with n_b rows and
context L_b sees keys 0 .. L_b - n_b + i.  Tolerance: max-abs 1.5e-2, mean-abs
2e-3 against fp64.
"""

import numpy as np
import pytest
import torch

from cases import oracle_compact, tiny_spec
from gpu_common import DEV, assert_close, no_device_errors, run_store
from paged_kv_cache_bf16_b200 import ops
from paged_kv_cache_bf16_b200 import workloads as W

pytestmark = pytest.mark.gpu

QLENS = [1, 2, 3, 4, 5, 8, 9, 16, 17, 40, 1, 2, 4, 4]


def _workload(seed, D, Hq, Hkv, BS, qlens, hi=3000):
    rng = W.SplitMix64(seed)
    qlens = np.array(qlens, dtype=np.int32)
    # contexts include the new rows; a few sequences are all new rows (L == n)
    ctx = np.array([n if i % 5 == 3 else rng.randint(int(n), hi) for i, n in enumerate(qlens)], dtype=np.int32)
    nblk = [-(-int(L) // BS) for L in ctx]
    spec = tiny_spec(name="multirow", seed=seed, head_dim=D, num_q_heads=Hq, num_kv_heads=Hkv, block_size=BS,
                     num_blocks=sum(nblk) + 4, num_seqs=len(qlens))
    perm = list(rng.permutation(spec.num_blocks))
    blocks = [np.array([perm.pop() for _ in range(k)], dtype=np.int64) for k in nblk]
    return W.Workload(spec=spec, ctx_lens0=ctx, query_lens=qlens, seq_blocks=blocks, max_blocks_per_seq=max(nblk))


CASES = [
    # (D, Hq, Hkv, block_size)
    (128, 16, 8, 256),
    (128, 32, 8, 256),
    (128, 64, 8, 16),
    (128, 8, 8, 32),
    (64, 8, 2, 16),
    (64, 16, 4, 128),
]


@pytest.mark.parametrize("hint", ["max", "one"])
@pytest.mark.parametrize("case", CASES, ids=lambda c: "D%d_q%d_kv%d_bs%d" % c)
def test_mixed_row_counts_in_one_call(case, hint):
    D, Hq, Hkv, BS = case
    wl = _workload(4000 + sum(case), D, Hq, Hkv, BS, QLENS)
    st = W.DeviceState(wl, DEV)
    run_store(st, 0)
    s = st.steps[0]
    # the hint picks the one- or two-tile decode variant; "one" under-states it,
    # which sends the longer short sequences to the tcgen05 kernel instead
    mq = int(wl.query_lens.max()) if hint == "max" else 1
    out = ops.paged_prefill_attention(s["q"], st.k_cache, st.v_cache, s["cu_seqlens_q"], mq, s["block_tables"],
                                      s["context_lens"])
    no_device_errors()
    ref, rows = oracle_compact(wl, 0)
    assert_close(out[torch.from_numpy(rows).to(DEV)], ref, f"{case} hint={hint}")


@pytest.mark.parametrize("n", [2, 4, 8])
def test_verify_rows_equal_single_row_problems(n):
    """Row i of an n-row verification sequence equals a decode of the same query over
    the first L - n + i + 1 tokens (bit-exact on the GPU is not required: the two run
    in different MMA columns; both are checked against the oracle)."""
    wl = _workload(4100 + n, 128, 16, 8, 256, [n] * 24, hi=2500)
    st = W.DeviceState(wl, DEV)
    run_store(st, 0)
    s = st.steps[0]
    out = ops.paged_prefill_attention(s["q"], st.k_cache, st.v_cache, s["cu_seqlens_q"], n, s["block_tables"],
                                      s["context_lens"])
    no_device_errors()
    L = wl.context_lens(0)
    cu = wl.cu_seqlens_q()
    # the same rows as decode problems over the truncated contexts
    dec_ctx = np.concatenate([np.arange(int(L[b]) - n + 1, int(L[b]) + 1) for b in range(wl.B)]).astype(np.int32)
    bt = np.repeat(wl.block_tables(0), n, axis=0)
    dec = ops.paged_decode_attention(s["q"], st.k_cache, st.v_cache, torch.from_numpy(bt).to(DEV),
                                     torch.from_numpy(dec_ctx).to(DEV))
    no_device_errors()
    ref, rows = oracle_compact(wl, 0)
    assert np.array_equal(rows, np.arange(int(cu[-1])))
    assert_close(out, ref, "verify rows")
    assert_close(dec, ref, "as decode rows")
