"""CPU tests of host-side logic: the layer schedule and the KV-footprint
figure against the pages (tests/golden), the workload parameters, and the
multi-process timing plumbing of bench.py (gloo, world size 2)."""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
GOLD = os.path.join(ROOT, "tests", "golden")


def _golden(name):
    rows = []
    for line in open(os.path.join(GOLD, name)):
        line = line.split("#", 1)[0].strip()
        if line:
            rows.append(line.split())
    return rows


@pytest.fixture(scope="module")
def pipeline():
    import importlib.util
    spec = importlib.util.spec_from_file_location("_hca_build",
                                                  os.path.join(ROOT, "long_context_attention_hca_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.build()
    from long_context_attention_hca_b200 import pipeline as p
    return p


def test_pro_schedule_matches_pages(pipeline):
    gold = {int(a): int(b) for a, b in _golden("pro_layer_schedule.txt")}
    assert len(gold) == 61
    ratios = pipeline.pro_layer_ratios(61)
    assert ratios == [gold[i] for i in range(61)]
    assert ratios.count(4) == 30 and ratios.count(128) == 31


def test_workload_parameters_match_pages():
    import hca_inputs as inp
    gold = {k: float(v) for k, v in _golden("page_parameters.txt")}
    for wl in inp.WORKLOADS.values():
        assert wl.m_csa == gold["csa_ratio"] and wl.m_hca == gold["hca_ratio"] and wl.W == gold["window"]
        if wl.d == 512:
            assert wl.c == gold["indexer_head_dim"]
    assert inp.WORKLOADS["decode_b4_1m"].k == gold["topk_pro"]
    assert inp.WORKLOADS["decode_b16_64k"].k == gold["topk_flash"]


def test_kv_footprint_is_about_two_percent_of_gqa8(pipeline):
    """The pages: the KV cache is about 2% of a bf16 GQA-8 (head dim 128)
    cache.  The stack workload's resident state against that baseline."""
    gold = {k: float(v) for k, v in _golden("page_parameters.txt")}
    B, T = 32, 262144
    ours = pipeline.kv_resident_bytes(B, T, pipeline.pro_layer_ratios(61))
    gqa = pipeline.gqa_bf16_bytes(B, T, 61)
    ratio = ours / gqa
    assert abs(ratio - gold["kv_ratio_vs_gqa8_bf16_hd128"]) < 0.005, ratio
    assert 43.0e9 < ours < 44.5e9


_CHILD = r"""
import os, sys, torch
sys.path.insert(0, os.environ["HCA_ROOT"])
import bench
world, rank, local, pg = bench.dist_setup(2)
v = bench.max_over_ranks(float(rank + 1) * 1.5, pg)
bench.barrier(pg)
assert v == 3.0, v
open(os.path.join(os.environ["HCA_OUT"], "rank%d" % rank), "w").write("ok %s" % v)
pg.destroy_process_group()
"""


def test_bench_max_over_ranks_gloo_world2(tmp_path):
    env = dict(os.environ, HCA_ROOT=ROOT, HCA_OUT=str(tmp_path), MASTER_ADDR="127.0.0.1", CUDA_VISIBLE_DEVICES="")
    script = tmp_path / "child.py"
    script.write_text(_CHILD)
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", "29533", str(script)]
    r = subprocess.run(cmd, env=env, capture_output=True, text=True, timeout=240)
    assert r.returncode == 0, r.stdout + r.stderr
    for rank in (0, 1):
        assert (tmp_path / f"rank{rank}").read_text() == "ok 3.0"


def test_decode_step_bytes_count_each_stream_once():
    """The decode step's algorithmic HBM bytes are the indexer's key stream
    plus the two attention calls (selected CSA entries, every HCA entry,
    windows, queries, outputs), each counted once: 95.68 MB at decode_b4_1m.
    The scores the top-k reads stay in L2 and are not part of the sum."""
    import bench
    import hca_inputs as inp
    wl = inp.WORKLOADS["decode_b4_1m"]
    algo = bench.decode_bytes(wl)
    assert set(algo) == {"indexer", "csa_attn", "hca_attn", "topk"}
    total = bench.step_bytes_of(algo)
    assert total == algo["indexer"] + algo["csa_attn"] + algo["hca_attn"]
    entry = 448 + 7 * 4 + 64 * 2
    assert entry == 604
    per_seq = (262144 * 68 + 4 * (64 + 4 + 4)) + (1024 * 604 + 128 * 1024 + 2 * 64 * 1024 + 1024 * 4) + \
              (8192 * 604 + 128 * 1024 + 2 * 64 * 1024)
    assert total == 4 * per_seq == 95683712


def test_prefill_attention_flops_counts_causal_keys():
    """Prefill attention work: 4*H*d flop per (query, key) over each query's
    causal key set; for the CSA call min(k, eligible) + window keys."""
    import bench
    import hca_inputs as inp
    import oracle
    wl = inp.WORKLOADS["prefill_4096_131k"]
    fl = bench.prefill_attn_flops(wl)
    n_csa = n_hca = 0
    for p in range(wl.t, wl.t + wl.Tq):
        e4, w0, w1 = oracle.causal_keys(p, 4, wl.W)
        e128, _, _ = oracle.causal_keys(p, 128, wl.W)
        n_csa += min(wl.k, len(e4)) + (w1 - w0)
        n_hca += len(e128) + (w1 - w0)
    assert fl["csa_attn"] == 4 * 64 * 512 * n_csa
    assert fl["hca_attn"] == 4 * 64 * 512 * n_hca
    att, _ = bench.prefill_flops(wl)
    assert att == fl["csa_attn"] + fl["hca_attn"]


def test_measured_traffic_only_for_its_workload_and_source():
    """A captured DRAM byte count is reported for the workload and the kernel
    source it was taken on, and for nothing else."""
    import bench
    assert bench.measured_traffic("hca_attn", "decode_b16_64k") is None
    assert bench.measured_traffic("csa_attn", "decode_b4_1m") is None
    for k, e in bench.MEASURED_TRAFFIC.items():
        got = bench.measured_traffic(k, e["workload"])
        assert got in (None, e["bytes"])


def test_dense_budget_beside_select(pipeline):
    """The HCA attention's default CTA cap in the decode step: the SMs that the
    select's B * floor(SMs / 2 / B) CTAs leave, never fewer than half."""
    dense_beside_select = pipeline.dense_beside_select
    assert dense_beside_select(148, 4) == 76         # select 4 x 18 = 72 CTAs
    assert dense_beside_select(148, 16) == 84        # 16 x 4 = 64
    assert dense_beside_select(148, 32) == 84        # 32 x 2 = 64
    assert dense_beside_select(148, 1) == 74         # 74 select CTAs: half
    assert dense_beside_select(148, 100) == 74       # one CTA per row would leave 48: half
    for sm in (132, 148, 160):
        for B in range(1, 200):
            c = dense_beside_select(sm, B)
            assert sm // 2 <= c <= sm
            sel = B * max(1, (sm // 2) // B)
            assert c == sm - sel or sel > sm - sm // 2
