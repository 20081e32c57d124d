"""Short multi-row sequences (speculative-decode verification, short chunks) in a
prefill call, against the fp64 oracle (GPU).

Sequences with g * n_b <= 16 query rows per KV head run on the split-KV decode
kernel's warp-level MMA tiles (one 8-column tile when the call's max_seqlen_q
bound says g * n_b <= 8, two otherwise); longer ones on the tcgen05 kernel.  A
bound that fits the decode tile runs that kernel alone.  Each
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


@pytest.mark.parametrize("case", CASES, ids=lambda c: "D%d_q%d_kv%d_bs%d" % c)
def test_mixed_row_counts_in_one_call(case):
    D, Hq, Hkv, BS = case
    wl = _workload(4000 + sum(case), D, Hq, Hkv, BS, QLENS)
    st = W.DeviceState(wl, DEV)
    run_store(st, 0)
    s = st.steps[0]
    mq = int(wl.query_lens.max())
    out = ops.paged_prefill_attention(s["q"], st.k_cache, st.v_cache, s["cu_seqlens_q"], mq, s["block_tables"],
                                      s["context_lens"])
    no_device_errors()
    ref, rows = oracle_compact(wl, 0)
    assert_close(out[torch.from_numpy(rows).to(DEV)], ref, f"{case}")


def _decode_rows_limit(g, max_seqlen_q):
    """Most query rows per sequence the decode kernel takes (its MMA columns)."""
    return 8 // g if max_seqlen_q * g <= 8 else 16 // g


@pytest.mark.parametrize("mq", [1, 2, 4])
@pytest.mark.parametrize("case", CASES, ids=lambda c: "D%d_q%d_kv%d_bs%d" % c)
def test_bound_within_decode_tile(case, mq):
    """max_seqlen_q <= m: the call runs the decode kernel alone.  Sequences within
    its m rows are exact; a longer one (the bound broken) reports
    NPV_DEVERR_QUERY_LENS and its rows are zeros."""
    D, Hq, Hkv, BS = case
    g = Hq // Hkv
    m = _decode_rows_limit(g, mq)
    if mq > m:
        pytest.skip("this bound sends long sequences to the tcgen05 kernel")
    wl = _workload(4200 + sum(case) + mq, D, Hq, Hkv, BS, QLENS)
    st = W.DeviceState(wl, DEV)
    run_store(st, 0)
    s = st.steps[0]
    out = ops.paged_prefill_attention(s["q"], st.k_cache, st.v_cache, s["cu_seqlens_q"], mq, s["block_tables"],
                                      s["context_lens"])
    long_seq = wl.query_lens > m
    assert long_seq.any()
    with pytest.raises(ops.NpvError) as ei:
        ops.check_device_errors()
    assert ei.value.bits == 0x8, ei.value.bits
    ref, rows = oracle_compact(wl, 0)
    cu = wl.cu_seqlens_q()
    owner = np.searchsorted(cu, rows, side="right") - 1
    keep = ~long_seq[owner]
    got = out[torch.from_numpy(rows).to(DEV)]
    assert_close(got[torch.from_numpy(keep).to(DEV)], ref[keep], f"{case} mq={mq} in-bound rows")
    dropped = got[torch.from_numpy(~keep).to(DEV)]
    assert dropped.numel() > 0 and torch.count_nonzero(dropped).item() == 0
    no_device_errors()


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


def test_malformed_query_ranges_on_decode_only_call():
    """With the decode kernel alone in the call, a cu_seqlens_q with a decreasing
    entry or a first entry other than 0 still sets NPV_DEVERR_QUERY_LENS, and the
    next call is exact."""
    wl = _workload(4300, 128, 16, 8, 256, [2, 1, 1, 4], hi=600)
    st = W.DeviceState(wl, DEV)
    run_store(st, 0)
    s = st.steps[0]
    for cu in ([0, 3, 2, 4, 8], [1, 2, 3, 4, 8], [0, 2, 3, 4, 7]):
        bad = torch.tensor(cu, dtype=torch.int32, device=DEV)
        ops.paged_prefill_attention(s["q"], st.k_cache, st.v_cache, bad, 4, s["block_tables"], s["context_lens"])
        with pytest.raises(ops.NpvError) as ei:
            ops.check_device_errors()
        assert ei.value.bits & 0x8, cu
    out = ops.paged_prefill_attention(s["q"], st.k_cache, st.v_cache, s["cu_seqlens_q"], 4, s["block_tables"],
                                      s["context_lens"])
    no_device_errors()
    ref, rows = oracle_compact(wl, 0)
    assert_close(out[torch.from_numpy(rows).to(DEV)], ref, "after malformed decode-only calls")
