"""npv_paged_prefill_attention (tcgen05 path + decode rows) against the fp64 oracle (GPU).

Chunked prefill: each sequence's n_b new rows are stored first, then attend
causally to all their cached context (bottom-right alignment).  Pools are
NaN-poisoned outside live tokens.  Tolerance: max-abs 1.5e-2, mean-abs 2e-3.
"""

import numpy as np
import pytest
import torch

from cases import oracle_compact, tiny_spec
from gpu_common import DEV, assert_close, no_device_errors, run_store
from paged_kv_cache_bf16_b200 import ops
from paged_kv_cache_bf16_b200 import workloads as W

pytestmark = pytest.mark.gpu


def run_prefill(st, step=0, **kw):
    s = st.steps[step]
    return ops.paged_prefill_attention(s["q"], st.k_cache, st.v_cache, s["cu_seqlens_q"], s["max_seqlen_q"],
                                       s["block_tables"], s["context_lens"], **kw)


def _check_full(spec):
    wl = W.draw(spec)
    st = W.DeviceState(wl, DEV)
    run_store(st, 0)
    out = run_prefill(st)
    no_device_errors()
    ref, rows = oracle_compact(wl, 0)
    assert_close(out[torch.from_numpy(rows).to(DEV)], ref, spec.name)
    return wl, st, out


def test_prefill_small_first():
    """One sequence, one 128-row tile, no prior context, D=128, g=2, BS=256."""
    _check_full(tiny_spec(name="p_small", seed=600, head_dim=128, num_q_heads=2, num_kv_heads=1, block_size=256,
                          num_blocks=4, num_seqs=1, prefill_seqs=1, prefill_len=64, prior_lo=0, prior_hi=0))


PREFILL_SHAPES = [
    # (D, Hq, Hkv, BS, prefill seqs, prefill_len, prior_hi, decode seqs, decode ctx_hi)
    (128, 16, 8, 256, 2, 300, 600, 4, 700),
    (128, 16, 8, 256, 3, 512, 1000, 0, 1),
    (128, 8, 8, 256, 2, 200, 300, 2, 100),
    (128, 32, 8, 256, 2, 100, 700, 3, 500),
    (128, 64, 8, 256, 1, 70, 400, 1, 90),
    (128, 16, 8, 32, 2, 150, 333, 3, 400),
    (128, 16, 4, 16, 2, 90, 150, 2, 200),
    (64, 8, 2, 16, 3, 77, 200, 2, 300),
    (64, 16, 4, 128, 2, 130, 500, 2, 260),
    (64, 8, 8, 256, 2, 129, 257, 1, 50),
    (128, 16, 8, 256, 2, 2, 10, 2, 30),
]


@pytest.mark.parametrize("shape", PREFILL_SHAPES,
                         ids=lambda s: "D%d_q%d_kv%d_bs%d_P%dx%d_prior%d_dec%d" % s[:8])
def test_prefill_shapes(shape):
    D, Hq, Hkv, BS, npre, plen, prior_hi, ndec, dec_hi = shape
    B = npre + ndec
    nb = npre * (-(-(prior_hi + plen) // BS)) + ndec * (-(-dec_hi // BS)) + 8
    spec = tiny_spec(name="p_shape", seed=700 + sum(shape), head_dim=D, num_q_heads=Hq, num_kv_heads=Hkv,
                     block_size=BS, num_blocks=nb, num_seqs=B, prefill_seqs=npre, prefill_len=plen, prior_lo=0,
                     prior_hi=prior_hi, ctx_lo=1, ctx_hi=dec_hi)
    _check_full(spec)


def test_prefill_prefix_shared_blocks():
    # groups of 2 sequences share their first 3 blocks; every sequence prefills
    spec = tiny_spec(name="p_prefix", seed=811, head_dim=128, num_q_heads=16, num_kv_heads=8, block_size=128,
                     num_blocks=200, num_seqs=4, prefill_seqs=4, prefill_len=150, prior_lo=400, prior_hi=700,
                     share_group=2, shared_blocks=3)
    _check_full(spec)


def test_prefill_chunk_split_matches_single_chunk():
    """A 384-row chunk equals a 256-row chunk followed by a 128-row chunk (on the GPU)."""
    spec = tiny_spec(name="p_split", seed=812, head_dim=128, num_q_heads=16, num_kv_heads=8, block_size=256,
                     num_blocks=40, num_seqs=1, prefill_seqs=1, prefill_len=384, prior_lo=700, prior_hi=700)
    wl = W.draw(spec)
    st = W.DeviceState(wl, DEV)
    run_store(st, 0)
    s = st.steps[0]
    full = run_prefill(st)
    L = int(wl.context_lens(0)[0])
    a = ops.paged_prefill_attention(s["q"][:256].contiguous(), st.k_cache, st.v_cache,
                                    torch.tensor([0, 256], dtype=torch.int32, device=DEV), 256, s["block_tables"],
                                    torch.tensor([L - 128], dtype=torch.int32, device=DEV))
    b = ops.paged_prefill_attention(s["q"][256:].contiguous(), st.k_cache, st.v_cache,
                                    torch.tensor([0, 128], dtype=torch.int32, device=DEV), 128, s["block_tables"],
                                    torch.tensor([L], dtype=torch.int32, device=DEV))
    no_device_errors()
    ref, _ = oracle_compact(wl, 0)
    assert_close(torch.cat([a, b]), ref, "split")
    assert_close(full, ref, "single")


def test_prefill_mixed_named_workload_all_rows():
    """The full chunked-prefill mix: 16 x 512-row chunks over priors up to 8,192 plus 240
    decode rows.  Every output row (8,192 prefill rows and 240 decode rows, all heads) is
    checked element by element against the fp64 oracle."""
    wl = W.workload("chunked_prefill_mixed")
    st = W.DeviceState(wl, DEV)
    run_store(st, 0)
    out = run_prefill(st)
    no_device_errors()
    dec = [b for b in range(wl.B) if wl.query_lens[b] == 1]
    ref, rows = oracle_compact(wl, 0, seqs=dec)
    assert_close(out[torch.from_numpy(rows).to(DEV)], ref, "decode rows")
    pre = [b for b in range(wl.B) if wl.query_lens[b] > 1]
    assert sum(int(wl.query_lens[b]) for b in pre) == 16 * 512
    ref, rows = oracle_compact(wl, 0, seqs=pre)
    assert_close(out[torch.from_numpy(rows).to(DEV)], ref, "prefill rows")


def test_prefill_spec_verify_named_workload():
    """Speculative-decode verification: 256 sequences x 4 query rows over priors up to 2,044,
    every row checked against the oracle."""
    wl = W.workload("spec_verify_decode")
    st = W.DeviceState(wl, DEV)
    run_store(st, 0)
    out = run_prefill(st)
    no_device_errors()
    ref, rows = oracle_compact(wl, 0)
    assert_close(out[torch.from_numpy(rows).to(DEV)], ref, "spec verify rows")


def test_prefill_decode_rows_equal_decode_call():
    """Rows with n_b == 1 inside a prefill call give the decode call's bits."""
    spec = tiny_spec(name="p_dec", seed=813, head_dim=128, num_q_heads=16, num_kv_heads=8, block_size=256,
                     num_blocks=60, num_seqs=9, prefill_seqs=0, ctx_lo=1, ctx_hi=1500)
    wl = W.draw(spec)
    st = W.DeviceState(wl, DEV)
    run_store(st, 0)
    s = st.steps[0]
    a = run_prefill(st)
    b = ops.paged_decode_attention(s["q"], st.k_cache, st.v_cache, s["block_tables"], s["context_lens"])
    no_device_errors()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_prefill_invalid_lengths_reported():
    spec = tiny_spec(name="p_bad", seed=814, head_dim=128, num_q_heads=16, num_kv_heads=8, block_size=256,
                     num_blocks=30, num_seqs=3, prefill_seqs=3, prefill_len=40, prior_lo=10, prior_hi=300)
    wl = W.draw(spec)
    st = W.DeviceState(wl, DEV)
    run_store(st, 0)
    s = st.steps[0]
    cl = s["context_lens"].clone()
    cl[1] = 10  # fewer tokens than the sequence's 40 new rows
    out = ops.paged_prefill_attention(s["q"], st.k_cache, st.v_cache, s["cu_seqlens_q"], s["max_seqlen_q"],
                                      s["block_tables"], cl)
    with pytest.raises(ops.NpvError) as ei:
        ops.check_device_errors()
    assert ei.value.bits & 0x4
    assert torch.count_nonzero(out[40:80]).item() == 0
    ref, rows = oracle_compact(wl, 0, seqs=[0, 2])
    assert_close(out[torch.from_numpy(rows).to(DEV)], ref, "valid sequences")


def test_prefill_malformed_query_ranges_reported():
    """cu_seqlens_q that does not partition q (a reversed entry, so ranges overlap, or a
    first entry other than 0) sets NPV_DEVERR_QUERY_LENS; the context stays usable."""
    spec = tiny_spec(name="p_cu", seed=815, head_dim=128, num_q_heads=16, num_kv_heads=8, block_size=256,
                     num_blocks=30, num_seqs=3, prefill_seqs=3, prefill_len=40, prior_lo=100, prior_hi=300)
    wl = W.draw(spec)
    st = W.DeviceState(wl, DEV)
    run_store(st, 0)
    s = st.steps[0]
    for cu in ([0, 80, 40, 120], [8, 48, 88, 120]):
        bad = torch.tensor(cu, dtype=torch.int32, device=DEV)
        ops.paged_prefill_attention(s["q"], st.k_cache, st.v_cache, bad, 80, s["block_tables"], s["context_lens"])
        with pytest.raises(ops.NpvError) as ei:
            ops.check_device_errors()
        assert ei.value.bits & 0x8, cu
    out = run_prefill(st)
    no_device_errors()
    ref, rows = oracle_compact(wl, 0)
    assert_close(out[torch.from_numpy(rows).to(DEV)], ref, "after malformed calls")
