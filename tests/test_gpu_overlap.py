"""GPU parity of the note's overlapped CSA compressor and the FP4
indexer-key compressor (section 7) against the CPU oracle, bit for bit:
FP8 codes, fp32 scales and bf16 RoPE dims of the entries; e2m1 code bytes
and ue8m0 exponents of the keys.  Also: keys compressed on the GPU and
scored by lightning_index give the oracle's scores of the oracle's keys."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import cache_host, host

pytestmark = pytest.mark.gpu

hca = pytest.importorskip("long_context_attention_hca_b200")

DEV = "cuda"


def _gen(seed):
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    return g


def _streams(B, T, d, seed):
    g = _gen(seed)
    return [torch.randn((B, T, d), generator=g, device=DEV).to(torch.bfloat16) for _ in range(4)]


@pytest.mark.parametrize("layout", [(128, 32, 32), (512, 64, 64)])
def test_csa_compress_overlap_bit_exact(layout):
    d, dr, g = layout
    B, n = 3, 41
    xa, za, xb, zb = _streams(B, 4 * n, d, 201)
    za[1, :8] = -1e4                                  # stream a switched off for two entries
    zb[2, 4:8] = 60.0                                 # saturating gates
    bias = torch.randn((8, d), generator=_gen(202), device=DEV) * 0.5
    cache = hca.KVCache(B, n, layout, zero=True)
    hca.csa_compress_overlap(xa, za, xb, zb, bias, n, cache)
    # a chunk of the same sequences from block k on, with stream a's block k-1 given
    k = 17
    cache2 = hca.KVCache(B, n, layout, zero=True)
    hca.csa_compress_overlap(xa[:, 4 * k:], za[:, 4 * k:], xb[:, 4 * k:], zb[:, 4 * k:], bias, n - k, cache2,
                             entry_begin=k, a_prev=xa[:, 4 * (k - 1):], za_prev=za[:, 4 * (k - 1):])
    torch.cuda.synchronize()
    c, s, r, worst = oracle.compress_overlap(host(xa), host(za), host(xb), host(zb), host(bias), 4, n, dr, g)
    assert worst < 1e-5
    gc, gs, gr = cache_host(cache)
    assert np.array_equal(gc, c)
    assert np.array_equal(gs.view(np.uint32), s.view(np.uint32))
    assert np.array_equal(gr, r)
    gc2, gs2, gr2 = cache_host(cache2)
    assert np.array_equal(gc2[:, k:], c[:, k:]) and np.array_equal(gs2[:, k:].view(np.uint32), s[:, k:].view(np.uint32))
    assert np.array_equal(gr2[:, k:], r[:, k:])


@pytest.mark.parametrize("c", [64, 128])
def test_indexer_key_compress_bit_exact_and_scores(c):
    B, n = 2, 301
    xa, za, xb, zb = _streams(B, 4 * n, c, 211)
    xb[0, :4, :32] = 0.0                              # an all-zero block: exponent byte 0, zero codes
    xa[1, 8:12] = xa[1, 8:12] * 1e-3                  # small values
    bias = torch.randn((8, c), generator=_gen(212), device=DEV) * 0.5
    kc = torch.zeros((B, n, c // 2), dtype=torch.uint8, device=DEV)
    ks = torch.zeros((B, n, c // 32), dtype=torch.uint8, device=DEV)
    hca.indexer_key_compress(xa, za, xb, zb, bias, n, kc, ks)
    torch.cuda.synchronize()
    wc, wsf = oracle.index_key_compress(host(xa), host(za), host(xb), host(zb), host(bias), 4, n)
    assert np.array_equal(host(ks), wsf)
    assert np.array_equal(host(kc), wc)
    # the compressed keys feed the indexer
    g = _gen(213)
    Hi = 4
    qc = torch.randint(0, 256, (B, 1, Hi, c // 2), generator=g, device=DEV, dtype=torch.uint8)
    qs = torch.randint(123, 128, (B, 1, Hi, c // 32), generator=g, device=DEV, dtype=torch.uint8)
    w = torch.rand((B, 1, Hi), generator=g, device=DEV)
    pos = torch.full((B, 1), 4 * n - 1, dtype=torch.int32, device=DEV)
    sc = hca.lightning_index(qc, qs, w, kc, ks, pos, 4)
    torch.cuda.synchronize()
    want, _ = oracle.index_scores(host(qc), host(qs), host(w), wc, wsf, host(pos), 4)
    assert np.array_equal(host(sc).view(np.uint32), want.view(np.uint32))
