"""compressed_attn_decode_noalloc against compressed_attn_decode.

The no-allocation entry point is for callers that cannot get device memory
when they call the library, e.g. a plug-in inside an engine that owns every
byte of device memory and allows no allocation after start-up, or a
latency-critical path that cannot take cudaMalloc's implicit device
synchronisation.  Its split-K scratch is a 16 MiB array built into the
library.  This test calls it through the C ABI twice in a row on different
inputs (a dense HCA-style call, then a sparse CSA-style call, so the second
call runs over the first call's leftover scratch) and checks each output
against the regular entry point with a caller workspace, within the
attention tolerance used everywhere else (bf16, max-abs 1e-2, mean-rel
1e-3).  It also checks that a request needing more scratch is refused
without launching anything.
"""
import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

hca = pytest.importorskip("long_context_attention_hca_b200")

DEV = "cuda"
_V, _I32, _F = ctypes.c_void_p, ctypes.c_int32, ctypes.c_float


def _fn():
    f = hca._lib.compressed_attn_decode_noalloc
    f.argtypes = [_V, _I32, _I32, hca.Layout, hca.CacheStruct, _V, _I32, _V, _I32, _V, _I32, _F, _V, _V, _V]
    f.restype = ctypes.c_int
    return f


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _cache(B, cap, seed):
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    c = hca.KVCache(B, cap, hca.LAYOUT_512)
    codes = torch.randint(0, 256, c.codes.shape, generator=g, device=DEV, dtype=torch.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0x38
    c.codes.copy_(codes)
    c.scales.copy_(torch.rand(c.scales.shape, generator=g, device=DEV) * 0.01 + 0.001)
    c.rope.copy_(torch.randn(c.rope.shape, generator=g, device=DEV).to(torch.bfloat16))
    return c, g


def _close(a, b):
    a = a.float().cpu().numpy().astype(np.float64)
    b = b.float().cpu().numpy().astype(np.float64)
    d = np.abs(a - b)
    return d.max() <= 1e-2 and d.sum() / max(np.abs(b).sum(), 1e-30) <= 1e-3


def test_noalloc_matches_regular_entry_point_twice():
    f = _fn()
    B, cap, W, H, d = 2, 5000, 128, 64, 512
    scale = d ** -0.5
    cache, g = _cache(B, cap, 7)
    # call 1: dense (every entry), long enough to need split-K scratch
    q1 = torch.randn((B, H, d), generator=g, device=DEV).to(torch.bfloat16)
    win1 = torch.randn((B, W, d), generator=g, device=DEV).to(torch.bfloat16)
    n1 = torch.tensor([cap, 3001], dtype=torch.int32, device=DEV)
    assert hca.decode_workspace_size(B, H, hca.LAYOUT_512, cap, W) > 0
    ref1 = hca.compressed_attn_decode(q1, cache, n1, cap, win1, scale)
    out1 = torch.empty_like(q1)
    lse1 = torch.empty((B, H), dtype=torch.float32, device=DEV)
    st = f(_p(q1), B, H, cache.c_layout, cache.c_struct, None, 0, _p(n1), cap, _p(win1), W, scale, _p(out1),
           _p(lse1), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == hca.HCA_OK, hca._lib.hca_status_string(st)
    # call 2: sparse selection with new queries and windows
    k = 1024
    q2 = torch.randn((B, H, d), generator=g, device=DEV).to(torch.bfloat16)
    win2 = torch.randn((B, W, d), generator=g, device=DEV).to(torch.bfloat16)
    idx = torch.full((B, k), -1, dtype=torch.int32, device=DEV)
    counts = [1024, 700]
    for b in range(B):
        idx[b, :counts[b]] = torch.randperm(cap, generator=g, device=DEV)[:counts[b]].sort().values.to(torch.int32)
    n2 = torch.tensor(counts, dtype=torch.int32, device=DEV)
    ref2 = hca.compressed_attn_decode(q2, cache, n2, k, win2, scale, idx=idx)
    out2 = torch.empty_like(q2)
    st = f(_p(q2), B, H, cache.c_layout, cache.c_struct, _p(idx), k, _p(n2), k, _p(win2), W, scale, _p(out2),
           None, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == hca.HCA_OK, hca._lib.hca_status_string(st)
    torch.cuda.synchronize()
    assert _close(out1, ref1)
    assert _close(out2, ref2)
    assert torch.all(torch.isfinite(lse1))


def test_noalloc_refuses_requests_beyond_its_scratch():
    """Under the default launch budget (one split per SM) the split-K scratch of
    any request stays below the 16 MiB array, so the budget is raised first to
    make a request that needs more."""
    f = _fn()
    B, cap, W, H, d = 8, 20000, 128, 64, 512
    prev = hca.set_launch_budget(hca.BUDGET_DENSE_DECODE, 1024)
    try:
        assert hca.decode_workspace_size(B, H, hca.LAYOUT_512, cap, W) > (16 << 20)
        cache, g = _cache(B, 8, 9)                       # pointers only; nothing may be launched
        q = torch.zeros((B, H, d), dtype=torch.bfloat16, device=DEV)
        win = torch.zeros((B, W, d), dtype=torch.bfloat16, device=DEV)
        n = torch.zeros((B,), dtype=torch.int32, device=DEV)
        out = torch.full((B, H, d), 7.0, dtype=torch.bfloat16, device=DEV)
        st = f(_p(q), B, H, cache.c_layout, cache.c_struct, None, 0, _p(n), cap, _p(win), W, d ** -0.5, _p(out),
               None, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    finally:
        hca.set_launch_budget(hca.BUDGET_DENSE_DECODE, prev)
    assert st == hca.HCA_ERR_SCRATCH_LIMIT
    torch.cuda.synchronize()
    assert torch.all(out == 7.0)
