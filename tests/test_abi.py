"""The C-ABI library: it loads, exports every declared symbol, validates on the host (CPU only).

No compute call is made: these run without a GPU.
"""

import ctypes as C
import subprocess
import sys

import pytest

from paged_kv_cache_bf16_b200 import build, ops


@pytest.fixture(scope="module")
def lib():
    build.build()
    return ops.lib()


def test_header_declares_the_three_calls():
    names = ops.exported_symbols()
    for n in ("npv_store_kvcache", "npv_paged_decode_attention", "npv_paged_prefill_attention",
              "npv_paged_decode_workspace_size", "npv_paged_prefill_workspace_size", "npv_check_device_errors",
              "npv_status_string", "npv_version"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    for n in ops.exported_symbols():
        assert hasattr(lib, n), n
    out = subprocess.run(["nm", "-D", "--defined-only", ops.LIB_PATH], capture_output=True, text=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    assert set(ops.exported_symbols()) <= exported
    # nothing else of ours leaks out of the shared object
    assert not [s for s in exported if s.startswith("_ZN3npv")]


def test_status_strings_and_version(lib):
    for code in range(6):
        assert lib.npv_status_string(code)
    assert lib.npv_status_string(99) == b"unknown status"
    assert lib.npv_version() >= 100


def test_host_validation_before_any_cuda_call(lib):
    # null pointers and bad shapes are rejected synchronously, with no device touched
    assert lib.npv_store_kvcache(None, None, 0, 0, None, None, None, 4, 8, 16, 2, 64, None) == 1
    assert lib.npv_store_kvcache(None, None, 0, 0, None, None, None, 0, 8, 16, 2, 64, None) == 0
    assert lib.npv_store_kvcache(None, None, 0, 0, None, None, None, -1, 8, 16, 2, 64, None) == 1
    assert lib.npv_paged_decode_attention(None, None, 0, None, None, None, 4, None, 2, 6, 4, 128, 8, 16, 0.0, None,
                                          0, None) == 1


def test_rope_store_host_validation(lib):
    f = lib.npv_rope_store_kvcache
    # (q, q_stride, Hq, key, value, k_stride, v_stride, positions, k_cache, v_cache, slots, T, NB, BS, Hkv, D,
    #  base, stream)
    ok = dict(T=0, D=64, base=1.0e6)

    def call(T=0, D=64, base=1.0e6, hq=2):
        return f(None, 0, hq, None, None, 0, 0, None, None, None, None, T, 8, 16, 2, D, base, None)

    assert call(**ok) == 0                   # no tokens: a no-op
    assert call(T=-1) == 1                   # negative count
    assert call(T=4) == 1                    # null pointers
    assert call(base=0.0) == 1               # the base must be positive and finite
    assert call(base=float("nan")) == 1
    assert call(base=float("inf")) == 1
    assert call(D=40) == 2                   # head_dim not a multiple of 16
    assert call(D=512) == 2                  # above 256
    assert call(hq=-1) == 1


def test_prefill_rejects_a_negative_row_bound(lib):
    assert lib.npv_paged_prefill_attention(None, None, None, -1, 8, None, None, None, 4, None, 2, 4, 2, 64, 8, 16,
                                           0.0, None, 0, None) == 1


def test_python_binding_fails_loudly_without_library(tmp_path, monkeypatch):
    code = ("import paged_kv_cache_bf16_b200.ops as o; o.LIB_PATH = %r\n"
            "try:\n    o.lib()\nexcept RuntimeError as e:\n    print('raised', e)\n") % str(tmp_path / "nope.so")
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, cwd=str(tmp_path.parent))
    assert "raised" in r.stdout or "raised" in r.stderr or r.returncode != 0
