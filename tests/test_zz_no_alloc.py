"""The allocation-free decode entry point (GPU).

npv_paged_decode_attention_noalloc serves callers that cannot allocate device
memory or pass a workspace (a plugin host that owns all device memory, or a path
where cudaMalloc's possible device synchronisation is not allowed); it takes
its scratch from a fixed array inside the library.  This test calls it through
the C ABI twice in a row, on two different workloads.  Each output must equal
npv_paged_decode_attention's (which runs the same kernels with a caller
workspace) bit for bit, so a stale read of what the previous call left in the
array would show, and must lie within the attention tolerance of the fp64
oracle.  The file is collected last so that a run stopping at the first failure
has already run every other test.
"""

import ctypes as C

import pytest
import torch

from cases import oracle_compact
from gpu_common import DEV, assert_close, no_device_errors, run_store
from paged_kv_cache_bf16_b200 import ops
from paged_kv_cache_bf16_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _noalloc_fn():
    l = ops.lib()
    f = l.npv_paged_decode_attention_noalloc
    p, i32 = C.c_void_p, C.c_int32
    f.argtypes = [p, p, C.c_int64, p, p, p, i32, p, i32, i32, i32, i32, i32, i32, C.c_float, p]
    f.restype = C.c_int
    return f


def _compare(name_or_spec):
    wl = W.workload(name_or_spec) if isinstance(name_or_spec, str) else W.draw(name_or_spec)
    st = W.DeviceState(wl, DEV)
    run_store(st, 0)
    s = st.steps[0]
    ref = ops.paged_decode_attention(s["q"], st.k_cache, st.v_cache, s["block_tables"], s["context_lens"])
    out = torch.full_like(ref, float("nan"))
    stream = torch.cuda.current_stream().cuda_stream
    rc = _noalloc_fn()(out.data_ptr(), s["q"].data_ptr(), s["q"].stride(0), st.k_cache.data_ptr(),
                       st.v_cache.data_ptr(), s["block_tables"].data_ptr(), s["block_tables"].shape[1],
                       s["context_lens"].data_ptr(), wl.B, wl.Hq, wl.Hkv, wl.D, wl.NB, wl.BS, 0.0, stream)
    assert rc == 0, ops.lib().npv_status_string(rc)
    no_device_errors()
    assert torch.equal(out.view(torch.int16), ref.view(torch.int16))
    want, rows = oracle_compact(wl, 0)
    assert_close(out[torch.from_numpy(rows).to(DEV)], want, wl.spec.name)


def test_noalloc_matches_workspace_entry_point_twice():
    torch.cuda.set_device(DEV)
    # first call: D=64, 4 Q / 2 KV heads, 16-token blocks
    _compare("tiny_decode")
    # second call reuses the scratch the first one left behind: D=128, 32 Q / 8 KV heads
    _compare(W.Spec(name="noalloc_second", seed=31, num_seqs=40, num_q_heads=32, num_kv_heads=8, head_dim=128,
                    block_size=256, num_blocks=400, ctx_lo=1, ctx_hi=3000))
