"""Shared pieces of the GPU parity tests (they call libnpv through its C ABI)."""

from __future__ import annotations

import numpy as np
import torch

from paged_kv_cache_bf16_b200 import ops
from paged_kv_cache_bf16_b200 import workloads as W

# Attention tolerance against the fp64 oracle: bf16 inputs, fp32 accumulation,
# one bf16 rounding of the output.
MAX_ABS = 1.5e-2
MEAN_ABS = 2e-3

DEV = "cuda:0"


def out_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to(torch.float64).cpu().numpy()


def assert_close(gpu: torch.Tensor, ref: np.ndarray, what: str = ""):
    g = out_f64(gpu)
    assert g.shape == ref.shape, (g.shape, ref.shape)
    assert np.isfinite(g).all(), f"{what}: non-finite output (a stray read of a poisoned slot?)"
    err = np.abs(g - ref)
    mx, mean = float(err.max()), float(err.mean())
    assert mx <= MAX_ABS and mean <= MEAN_ABS, f"{what}: max-abs {mx:.3e} mean-abs {mean:.3e}"
    return mx, mean


def no_device_errors():
    bits = ops.check_device_errors()
    assert bits == 0


def run_store(state: W.DeviceState, step: int):
    s = state.steps[step]
    ops.store_kvcache(s["key"], s["value"], state.k_cache, state.v_cache, s["slot_mapping"])


def run_decode(state: W.DeviceState, step: int, **kw):
    s = state.steps[step]
    return ops.paged_decode_attention(s["q"], state.k_cache, state.v_cache, s["block_tables"], s["context_lens"],
                                      **kw)
