"""Shared pieces of the head-sharded o_proj tests (CPU and GPU)."""

from __future__ import annotations

import numpy as np

from cases import tiny_spec
from paged_kv_cache_bf16_b200 import workloads as W

HIDDEN = 1024  # Qwen3-0.6B's hidden size (16 query heads x 128 = 2048 o_proj inputs)


def tp_workload(seed: int = 8100, num_seqs: int = 12, hq: int = 16, hkv: int = 8, d: int = 128):
    return W.draw(tiny_spec(name="tp_decode", seed=seed, num_seqs=num_seqs, num_q_heads=hq, num_kv_heads=hkv,
                            head_dim=d, block_size=16, num_blocks=num_seqs * 40 + 8, ctx_lo=1, ctx_hi=600))


def oproj_weight(seed: int, hidden: int, k: int) -> np.ndarray:
    """W_o [hidden, k] as bf16 bits, entries N(0, 1/k)."""
    rng = np.random.default_rng(seed)
    return W.f32_to_bf16_bits((rng.standard_normal((hidden, k)) / np.sqrt(k)).astype(np.float32))


def oproj_bound(a_f64: np.ndarray, w_f64: np.ndarray, partials_abs: np.ndarray, y_ref: np.ndarray) -> np.ndarray:
    """Per-element error bound of the row-parallel o_proj against the fp64 product of the
    same bf16 inputs: each rank's partial is rounded once to bf16 (at most 2^-8 of it,
    bf16 having 8 significant bits) and the result once more (2^-8 of it), plus fp32
    accumulation (2^-24 per term over at most 2^11 terms, bounded by 2^-12 of the sum
    of |a w|)."""
    abs_terms = np.abs(a_f64) @ np.abs(w_f64).T
    return 2.0 ** -8 * (partials_abs + np.abs(y_ref)) + 2.0 ** -12 * abs_terms + 1e-7
