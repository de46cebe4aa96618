"""hca_decode_step_host, the C ABI's host-to-host decode step (one CSA and
one HCA layer: query copies in, index + top-k, both attention calls, output
copies out), called through ctypes with pinned host buffers (the indexer
query as three arrays and the outputs apart, or each packed back to back
for one copy): its outputs are
those of the device-resident step bit for bit, and the oracle's within the
attention tolerance, on tiny_decode_1k and decode_b16_64k; the step also
runs captured in a CUDA graph."""
import numpy as np
import pytest
import torch

import hca_inputs as inp
import oracle
from gpu_util import assert_attn_close, cache_host, host

pytestmark = pytest.mark.gpu

hca = pytest.importorskip("long_context_attention_hca_b200")
from hca_workloads import build_decode  # noqa: E402
from long_context_attention_hca_b200.pipeline import DecodeRunner, packed_indexer_query  # noqa: E402


@pytest.mark.parametrize("name,packed", [("tiny_decode_1k", False), ("decode_b16_64k", False),
                                         ("tiny_decode_1k", True)])
def test_step_host_capi(name, packed):
    wl = inp.WORKLOADS[name]
    dw = build_decode(wl)
    runner = DecodeRunner(dw.layers, wl.B, wl.H, wl.k, wl.t, wl.softmax_scale)
    ref = [o.clone() for o in runner.step(dw.q, dw.iq)]
    torch.cuda.synchronize()
    h_q = [t.to("cpu").pin_memory() for t in dw.q]
    if packed:      # the indexer query's three arrays back to back: one copy
        h_iq = [None if t is None else packed_indexer_query(t, device="cpu", pin=True) for t in dw.iq]
    else:
        h_iq = [None if t is None else tuple(x.to("cpu").pin_memory() for x in t) for t in dw.iq]
    if packed:      # and both outputs back to back: one copy
        h_out = list(torch.zeros((len(runner.out),) + tuple(runner.out[0].shape), dtype=runner.out[0].dtype,
                                 pin_memory=True).unbind(0))
    else:
        h_out = [torch.zeros_like(o, device="cpu").pin_memory() for o in runner.out]
    d_q = [torch.zeros_like(t) for t in dw.q]
    if packed:
        d_iq = [None if t is None else tuple(x.zero_() for x in packed_indexer_query(t)) for t in dw.iq]
    else:
        d_iq = [None if t is None else tuple(torch.zeros_like(x) for x in t) for t in dw.iq]
    for o in runner.out:
        o.zero_()
    plan = runner.capi_plan(d_q, d_iq, packed=3 if packed else 0)
    runner.step_host_capi(plan, h_q, h_iq, h_out)
    torch.cuda.synchronize()
    for a, b in zip(h_out, ref):
        assert torch.equal(a.view(torch.int16), b.cpu().view(torch.int16))
    # against the oracle: top-k set of the CSA layer and both outputs
    for li, L in enumerate(dw.layers):
        codes, scales, rope = cache_host(L.cache)
        for b in range(wl.B):
            if L.ratio == 4:
                qc, qs, w = (host(t) for t in dw.iq[li])
                pos = np.array([[wl.t]], np.int32)
                s, _ = oracle.index_scores(qc[b:b + 1], qs[b:b + 1], w[b:b + 1], host(L.k_codes)[b:b + 1],
                                           host(L.k_sf)[b:b + 1], pos, 4)
                idx, cnt = oracle.topk(s[0], pos[0], 4, wl.k)
                ent = idx[0, :cnt[0]]
            else:
                ent = np.arange(L.n_entries)
            want, _ = oracle.attend(host(dw.q[li])[b], codes[b], scales[b], rope[b], ent, host(L.window)[b],
                                    wl.softmax_scale, wl.g)
            assert_attn_close(host(h_out[li])[b], want, f"{name} layer {li} b {b}")
    # the same call captured in a graph and replayed
    for h in h_out:
        h.zero_()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        runner.step_host_capi(plan, h_q, h_iq, h_out)
    g.replay()
    torch.cuda.synchronize()
    for a, b in zip(h_out, ref):
        assert torch.equal(a.view(torch.int16), b.cpu().view(torch.int16))
