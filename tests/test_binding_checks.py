"""The Python binding refuses host tensors, tensors split over devices and non-bf16
activations before anything reaches the C ABI (CPU: no GPU is touched)."""

import pytest
import torch

from paged_kv_cache_bf16_b200 import ops


def _cpu_args():
    q = torch.zeros((2, 4, 64), dtype=torch.bfloat16)
    kc = torch.zeros((8, 16, 2, 64), dtype=torch.bfloat16)
    bt = torch.zeros((2, 4), dtype=torch.int32)
    cl = torch.ones(2, dtype=torch.int32)
    return q, kc, kc.clone(), bt, cl


def test_host_tensors_are_refused():
    q, kc, vc, bt, cl = _cpu_args()
    with pytest.raises(ValueError, match="CUDA tensor"):
        ops.paged_decode_attention(q, kc, vc, bt, cl)
    with pytest.raises(ValueError, match="CUDA tensor"):
        ops.store_kvcache(q, q, kc, vc, torch.zeros(2, dtype=torch.int32))
    with pytest.raises(ValueError, match="CUDA tensor"):
        ops.store_kvcache_and_decode_attention(q, q[:, :2], q[:, :2], kc, vc, torch.zeros(2, dtype=torch.int32),
                                               bt, cl)
    with pytest.raises(ValueError, match="CUDA tensor"):
        ops.paged_prefill_attention(q, kc, vc, torch.tensor([0, 1, 2], dtype=torch.int32), 1, bt, cl)


class _LooksCuda(torch.Tensor):
    """A host tensor that reports itself as CUDA, to reach the dtype rule without a GPU."""

    @property
    def is_cuda(self):
        return True


def _looks_cuda(t):
    return torch.Tensor._make_subclass(_LooksCuda, t)


def test_dtype_rule_is_bf16_for_activations_and_caches():
    q16 = _looks_cuda(torch.zeros(4, dtype=torch.float16))
    qbf = _looks_cuda(torch.zeros(4, dtype=torch.bfloat16))
    idx = _looks_cuda(torch.zeros(4, dtype=torch.int32))
    with pytest.raises(TypeError, match="bfloat16"):
        ops._on_one_gpu("x", bf16=[("q", q16)], other=[("block_tables", idx)])
    assert ops._on_one_gpu("x", bf16=[("q", qbf), ("out", None)], other=[("block_tables", idx)]) is None
    # a host tensor among device ones is named
    with pytest.raises(ValueError, match="context_lens"):
        ops._on_one_gpu("x", bf16=[("q", qbf)], other=[("context_lens", torch.zeros(2, dtype=torch.int32))])
