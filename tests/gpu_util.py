"""Helpers for the GPU parity tests: host copies for the oracle and the
floating-point tolerance of the attention outputs.

Tolerance (attention outputs, bf16): the GPU output against the oracle's
fp64 result rounded to bf16 must satisfy max |a - b| <= 1e-2 and
sum |a - b| / sum |b| <= 1e-3 (the bar the workloads are specified with).
Codes, scales, index scores and top-k sets are compared bit for bit.
"""
from __future__ import annotations

import os

import numpy as np
import torch

import oracle

MAX_ABS = 1e-2
MEAN_REL = 1e-3


def host(t: torch.Tensor) -> np.ndarray:
    t = t.detach().to("cpu").contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    return oracle.bf16_to_f32(bits).astype(np.float64)


def attn_errors(gpu_bits: np.ndarray, ref64: np.ndarray):
    a = bf16_to_f64(gpu_bits)
    b = bf16_to_f64(oracle.round_bf16(ref64))
    diff = np.abs(a - b)
    return float(diff.max()), float(diff.sum() / max(np.abs(b).sum(), 1e-30))


def assert_attn_close(gpu_bits, ref64, what=""):
    mx, mr = attn_errors(gpu_bits, ref64)
    log = os.environ.get("HCA_ATTN_ERROR_LOG")
    if log:                                   # margin report: one line per comparison
        with open(log, "a") as f:
            f.write(f"{os.environ.get('PYTEST_CURRENT_TEST', '?').split(' ')[0]} {what} max_abs={mx:.3e} mean_rel={mr:.3e}\n")
    assert mx <= MAX_ABS and mr <= MEAN_REL, f"{what}: max-abs {mx:.3e} (<= {MAX_ABS}), mean-rel {mr:.3e} (<= {MEAN_REL})"
    return mx, mr


def cache_host(cache, b=None):
    """(codes, scales, rope) numpy of one sequence (b) or all."""
    sl = slice(None) if b is None else b
    return host(cache.codes[sl]), host(cache.scales[sl]), host(cache.rope[sl])
