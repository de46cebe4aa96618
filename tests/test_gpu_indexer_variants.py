"""GPU parity of the note's indexer variants ("DeepSeek V4 ..." reading note,
section 7 parameters: n_h^I = 64 indexer heads; section 9: the top-k
selector's index scores in BF16 instead of FP32), bit for bit against the
oracle: 64-head scores (the same ordered fp32 head sum), BF16 scores (the
fp32 score rounded once to bf16, nearest even) and top-k sets over BF16
scores (the same total order: value descending, lower index first, which
BF16's many ties exercise)."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import host

pytestmark = pytest.mark.gpu

hca = pytest.importorskip("long_context_attention_hca_b200")

DEV = "cuda"


def _gen(seed):
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    return g


def _inputs(B, Tq, Hi, Nc, seed, c=128):
    g = _gen(seed)
    qc = torch.randint(0, 256, (B, Tq, Hi, c // 2), generator=g, device=DEV, dtype=torch.uint8)
    qs = torch.randint(123, 128, (B, Tq, Hi, c // 32), generator=g, device=DEV, dtype=torch.uint8)
    w = torch.rand((B, Tq, Hi), generator=g, device=DEV)
    kc = torch.randint(0, 256, (B, Nc, c // 2), generator=g, device=DEV, dtype=torch.uint8)
    ks = torch.randint(123, 128, (B, Nc, c // 32), generator=g, device=DEV, dtype=torch.uint8)
    return qc, qs, w, kc, ks


def _bf16_bits(scores_f32):
    return oracle.f32_to_bf16(scores_f32)


@pytest.mark.parametrize("Hi,score_bf16", [(64, False), (64, True), (4, True)])
def test_index_scores_variants(Hi, score_bf16):
    B, Tq, Nc, m = 2, 3, 3000, 4          # the tensor-map path: Nc a multiple of 4
    qc, qs, w, kc, ks = _inputs(B, Tq, Hi, Nc, 300 + Hi)
    pos = torch.tensor([[4 * Nc, 77, 4 * (Nc // 2) - 1], [3, 4 * Nc - 5, 1 << 30]], dtype=torch.int32, device=DEV)
    s = hca.lightning_index(qc, qs, w, kc, ks, pos, m, score_bf16=score_bf16)
    torch.cuda.synchronize()
    want, n_inexact = oracle.index_scores(host(qc), host(qs), host(w), host(kc), host(ks), host(pos), m)
    assert n_inexact == 0
    if score_bf16:
        assert np.array_equal(host(s), _bf16_bits(want))
    else:
        assert np.array_equal(host(s).view(np.uint32), want.view(np.uint32))


@pytest.mark.parametrize("Hi", [4, 64])
def test_fused_select_bf16_and_64_heads(Hi):
    """Decode shape: one query per sequence over a long row (histogram path)."""
    B, Nc, m, k = 2, 40000, 4, 512
    qc, qs, w, kc, ks = _inputs(B, 1, Hi, Nc, 310 + Hi)
    pos = torch.tensor([4 * Nc - 1, 4 * 30001 + 2], dtype=torch.int32, device=DEV)
    for bf in (False, True):
        sc, idx, cnt = hca.lightning_index_topk(qc, qs, w, kc, ks, pos, m, k, score_bf16=bf)
        torch.cuda.synchronize()
        want, _ = oracle.index_scores(host(qc), host(qs), host(w), host(kc), host(ks), host(pos).reshape(B, 1), m)
        if bf:
            wb = _bf16_bits(want)
            assert np.array_equal(host(sc), wb)
            vals = oracle.bf16_to_f32(wb[:, 0])
        else:
            assert np.array_equal(host(sc).view(np.uint32), want.view(np.uint32))
            vals = want[:, 0]
        ri, rc = oracle.topk(vals, host(pos), m, k)
        assert np.array_equal(host(cnt), rc) and np.array_equal(host(idx), ri), f"bf16={bf}"


def test_topk_bf16_ties_and_signed_zero():
    R, Nc, k = 3, 20000, 700
    g = _gen(320)
    vals = (torch.randn((R, Nc), generator=g, device=DEV) * 0.5).to(torch.bfloat16)
    vals[0, ::3] = 0.0                                             # +0 and -0 tie as values
    vals[0, 1::7] = -0.0
    vals[1] = torch.tensor(1.5, dtype=torch.bfloat16)              # one value everywhere: the lowest indices win
    vals[2, 5000:] = float("-inf")
    pos = torch.tensor([4 * Nc - 1, 4 * Nc - 1, 4 * 9000 - 1], dtype=torch.int32, device=DEV)
    idx, cnt = hca.topk_select(vals, pos, 4, k)
    torch.cuda.synchronize()
    ri, rc = oracle.topk(oracle.bf16_to_f32(host(vals)), host(pos), 4, k)
    assert np.array_equal(host(cnt), rc) and np.array_equal(host(idx), ri)
    assert np.array_equal(host(idx)[1], np.arange(k))
