"""npv_store_kvcache against the oracle's store: bit-exact, whole pools (GPU)."""

import numpy as np
import pytest
import torch

from cases import tiny_spec
from gpu_common import DEV, no_device_errors
from oracle import oracle as O
from paged_kv_cache_bf16_b200 import ops
from paged_kv_cache_bf16_b200 import workloads as W

pytestmark = pytest.mark.gpu

SMALL = {
    "tiny_decode": W.SPECS["tiny_decode"],
    "mixed_d64_bs16": tiny_spec(seed=11, head_dim=64, block_size=16, num_blocks=200, num_seqs=9, prefill_seqs=3,
                                prefill_len=37, prior_lo=0, prior_hi=70, ctx_lo=1, ctx_hi=90),
    "mixed_d128_bs256": tiny_spec(seed=12, head_dim=128, block_size=256, num_blocks=40, num_seqs=7,
                                  num_q_heads=16, num_kv_heads=8, prefill_seqs=2, prefill_len=300, prior_lo=0,
                                  prior_hi=600, ctx_lo=1, ctx_hi=700),
    "hkv1_d128_bs32": tiny_spec(seed=13, head_dim=128, block_size=32, num_blocks=64, num_seqs=5, num_q_heads=4,
                                num_kv_heads=1, ctx_lo=1, ctx_hi=200),
}


def _device_pools(kp, vp):
    return W.bits_to_torch(kp, DEV), W.bits_to_torch(vp, DEV)


@pytest.mark.parametrize("name", sorted(SMALL))
def test_store_whole_pool_bit_exact(name):
    wl = W.draw(SMALL[name])
    kp, vp = wl.host_pool()
    kd, vd = _device_pools(kp, vp)
    k, v = wl.new_kv(0)
    slots = wl.slot_mapping(0)
    ops.store_kvcache(W.bits_to_torch(k, DEV), W.bits_to_torch(v, DEV), kd, vd, torch.from_numpy(slots).to(DEV))
    no_device_errors()
    O.store_kvcache(k, v, kp, vp, slots)
    assert np.array_equal(W.torch_to_bits(kd), kp)
    assert np.array_equal(W.torch_to_bits(vd), vp)


@pytest.mark.parametrize("name", sorted(W.SPECS))
def test_store_named_workload_bit_exact(name):
    """Full-size workloads: every block the store touches, plus a sample of the rest."""
    wl = W.workload(name)
    st = W.DeviceState(wl, DEV)
    s = st.steps[0]
    slots = wl.slot_mapping(0)
    touched = np.unique(slots // wl.BS)
    rng = np.random.default_rng(0)
    others = np.setdiff1d(rng.choice(wl.NB, size=min(wl.NB, 256), replace=False), touched)
    idx_t = torch.from_numpy(touched).to(DEV)
    idx_o = torch.from_numpy(others).to(DEV)
    before_k = W.torch_to_bits(st.k_cache[idx_t])
    before_v = W.torch_to_bits(st.v_cache[idx_t])
    other_k = W.torch_to_bits(st.k_cache[idx_o])
    other_v = W.torch_to_bits(st.v_cache[idx_o])
    ops.store_kvcache(s["key"], s["value"], st.k_cache, st.v_cache, s["slot_mapping"])
    no_device_errors()
    # the oracle stores into the host copy of the touched blocks (relabelled)
    pos = {int(p): i for i, p in enumerate(touched)}
    cslots = np.array([pos[int(x) // wl.BS] * wl.BS + int(x) % wl.BS for x in slots], dtype=np.int32)
    k, v = wl.new_kv(0)
    O.store_kvcache(k, v, before_k, before_v, cslots)
    assert np.array_equal(W.torch_to_bits(st.k_cache[idx_t]), before_k)
    assert np.array_equal(W.torch_to_bits(st.v_cache[idx_t]), before_v)
    assert np.array_equal(W.torch_to_bits(st.k_cache[idx_o]), other_k)
    assert np.array_equal(W.torch_to_bits(st.v_cache[idx_o]), other_v)
    del st
    torch.cuda.empty_cache()


def test_store_padding_and_out_of_range_slots():
    wl = W.draw(SMALL["mixed_d64_bs16"])
    kp, vp = wl.host_pool()
    kd, vd = _device_pools(kp, vp)
    k, v = wl.new_kv(0)
    slots = wl.slot_mapping(0).copy()
    slots[::5] = -1  # padding rows write nothing
    slots[3] = wl.NB * wl.BS  # out of range: reported, skipped
    ops.store_kvcache(W.bits_to_torch(k, DEV), W.bits_to_torch(v, DEV), kd, vd, torch.from_numpy(slots).to(DEV))
    with pytest.raises(ops.NpvError) as ei:
        ops.check_device_errors()
    assert ei.value.bits & 0x1
    assert ops.check_device_errors() == 0  # the check cleared the word
    slots_oracle = slots.copy()
    slots_oracle[3] = -1
    O.store_kvcache(k, v, kp, vp, slots_oracle)
    assert np.array_equal(W.torch_to_bits(kd), kp)
    assert np.array_equal(W.torch_to_bits(vd), vp)


def test_store_from_strided_qkv_slices():
    wl = W.draw(SMALL["mixed_d128_bs256"])
    kp, vp = wl.host_pool()
    kd, vd = _device_pools(kp, vp)
    k, v = wl.new_kv(0)
    T, Hkv, D, Hq = k.shape[0], wl.Hkv, wl.D, wl.Hq
    qkv = torch.zeros((T, (Hq + 2 * Hkv) * D), dtype=torch.bfloat16, device=DEV)
    qkv[:, Hq * D:(Hq + Hkv) * D] = W.bits_to_torch(k, DEV).reshape(T, -1)
    qkv[:, (Hq + Hkv) * D:] = W.bits_to_torch(v, DEV).reshape(T, -1)
    key = qkv[:, Hq * D:(Hq + Hkv) * D].view(T, Hkv, D)
    value = qkv[:, (Hq + Hkv) * D:].view(T, Hkv, D)
    assert key.stride(0) == (Hq + 2 * Hkv) * D
    slots = wl.slot_mapping(0)
    ops.store_kvcache(key, value, kd, vd, torch.from_numpy(slots).to(DEV))
    no_device_errors()
    O.store_kvcache(k, v, kp, vp, slots)
    assert np.array_equal(W.torch_to_bits(kd), kp)
    assert np.array_equal(W.torch_to_bits(vd), vp)


def test_store_empty_and_host_validation():
    kd = torch.zeros((4, 16, 2, 64), dtype=torch.bfloat16, device=DEV)
    vd = torch.zeros_like(kd)
    e = torch.zeros((0, 2, 64), dtype=torch.bfloat16, device=DEV)
    ops.store_kvcache(e, e, kd, vd, torch.zeros(0, dtype=torch.int32, device=DEV))
    key = torch.ones((3, 2, 64), dtype=torch.bfloat16, device=DEV)
    slots = torch.tensor([0, 1, 2], dtype=torch.int32, device=DEV)
    l = ops.lib()
    # misaligned source pointer
    rc = l.npv_store_kvcache(key.data_ptr() + 2, key.data_ptr(), 128, 128, kd.data_ptr(), vd.data_ptr(),
                             slots.data_ptr(), 3, 4, 16, 2, 64, None)
    assert rc == 1
    # stride smaller than a row
    rc = l.npv_store_kvcache(key.data_ptr(), key.data_ptr(), 64, 128, kd.data_ptr(), vd.data_ptr(),
                             slots.data_ptr(), 3, 4, 16, 2, 64, None)
    assert rc == 1
    assert torch.count_nonzero(kd).item() == 0
    no_device_errors()
