"""The decode kernel's bounded pipeline waits give up, report, and leave the
context usable (GPU).

A host-set test hook (npv_debug_inject_decode_timeout) leaves the first
pipeline stage of every CTA unfilled, so the consumer warps wait for a stage
that nothing fills; with the hook on, that wait gives up after about a
millisecond, while the producer's own waits keep their 2 s limit.  Nothing
faults or hangs: the call must end by itself, npv_check_device_errors must
report NPV_DEVERR_TIMEOUT, and the next call without the hook must match the
fp64 oracle.
"""

import time

import pytest
import torch

from cases import oracle_compact, tiny_spec
from gpu_common import DEV, assert_close, no_device_errors, run_decode, run_store
from paged_kv_cache_bf16_b200 import ops
from paged_kv_cache_bf16_b200 import workloads as W

pytestmark = pytest.mark.gpu


def test_decode_wait_gives_up_and_context_stays_usable():
    # ~20 chunks per CTA: producers also meet their own (2 s) wait for a stage the
    # consumers never release, and leave through their drain
    spec = tiny_spec(name="timeout", seed=950, head_dim=128, num_q_heads=16, num_kv_heads=8, block_size=256,
                     num_blocks=220, num_seqs=16, ctx_lo=2000, ctx_hi=3000)
    wl = W.draw(spec)
    st = W.DeviceState(wl, DEV)
    run_store(st, 0)
    no_device_errors()
    try:
        ops.inject_decode_timeout(True)
        t0 = time.time()
        run_decode(st, 0)
        with pytest.raises(ops.NpvError) as ei:
            ops.check_device_errors()
        elapsed = time.time() - t0
        assert ei.value.bits & 0x10, ei.value.bits
        assert elapsed < 30.0
    finally:
        ops.inject_decode_timeout(False)
    torch.cuda.synchronize()
    out = run_decode(st, 0)
    no_device_errors()
    ref, rows = oracle_compact(wl, 0)
    assert_close(out[torch.from_numpy(rows).to(DEV)], ref, "after the timeout")
