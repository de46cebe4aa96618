"""CPU tests of the C-ABI library: it loads, exports every symbol the header
declares, and rejects bad arguments on the host before touching the GPU
(these calls return before any CUDA call, so they run without a device)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "hca.h")


def _build_lib():
    import importlib.util
    spec = importlib.util.spec_from_file_location("_hca_build",
                                                  os.path.join(ROOT, "long_context_attention_hca_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod.build()


@pytest.fixture(scope="module")
def lib():
    return ctypes.CDLL(_build_lib())


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s+([a-z_][a-z0-9_]*)\s*\(", src, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_six_calls():
    names = declared_functions()
    for n in ("csa_compress", "hca_compress", "lightning_index", "topk_select", "compressed_attn_decode",
              "compressed_attn_prefill"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for n in declared_functions():
        assert hasattr(lib, n), n


def test_status_strings(lib):
    lib.hca_status_string.restype = ctypes.c_char_p
    assert lib.hca_status_string(0) == b"ok"
    assert lib.hca_status_string(1) == b"invalid argument"
    assert lib.hca_status_string(4) == b"workspace missing or too small"


class Layout(ctypes.Structure):
    _fields_ = [("d", ctypes.c_int32), ("d_rope", ctypes.c_int32), ("scale_group", ctypes.c_int32)]


class Cache(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("rope", ctypes.c_void_p),
                ("capacity", ctypes.c_int64)]


def test_host_validation_without_gpu(lib):
    V, I32, I64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
    lib.csa_compress.argtypes = [V, V, I64, V, I32, I64, Layout, Cache, I64, V]
    good = Layout(512, 64, 64)
    cache = Cache(None, None, None, 10)
    # unsupported layout is reported before pointers are looked at
    assert lib.csa_compress(None, None, 8, None, 1, 1, Layout(256, 64, 64), cache, 0, None) == 2
    # null pointers
    assert lib.csa_compress(None, None, 8, None, 1, 1, good, cache, 0, None) == 1
    # misaligned pointer
    assert lib.csa_compress(V(0x1008), V(0x1000), 8, V(0x1000), 1, 1, good,
                            Cache(0x1000, 0x1000, 0x1000, 10), 0, None) == 1
    # empty work is a no-op
    assert lib.csa_compress(None, None, 0, None, 0, 0, good, cache, 0, None) == 0
    lib.lightning_index.argtypes = [V, V, V, V, V, V, I32, I32, I64, I32, I32, I32, V, V]
    assert lib.lightning_index(None, None, None, None, None, None, 1, 1, 10, 4, 96, 4, None, None) == 2  # c
    assert lib.lightning_index(None, None, None, None, None, None, 1, 1, 10, 9, 128, 4, None, None) == 2  # Hi
    assert lib.lightning_index(None, None, None, None, None, None, 1, 1, 10, 4, 128, 0, None, None) == 1  # m
    lib.topk_select.argtypes = [V, V, I32, I64, I32, I32, V, V, V, ctypes.c_size_t, V]
    assert lib.topk_select(None, None, 1, 100, 4, 0, None, None, None, 0, None) == 2       # k = 0
    # a row longer than 2^19 scores needs the workspace path
    assert lib.topk_select(V(0x1000), V(0x1000), 1, 1 << 20, 4, 8, V(0x1000), V(0x1000), None, 0, None) == 4
    lib.topk_select_workspace_size.argtypes = [I32, I64, I32]
    lib.topk_select_workspace_size.restype = ctypes.c_size_t
    assert lib.topk_select_workspace_size(4, 262144, 1024) >= 4 * 262144 * 8   # few long rows: histogram path
    assert lib.topk_select_workspace_size(4096, 33000, 512) == 0               # many rows: clusters, no workspace
    assert lib.topk_select(None, None, 1, 100, 4, 8, None, None, None, 0, None) == 1       # null pointers
    lib.compressed_attn_decode.argtypes = [V, I32, I32, Layout, Cache, V, I32, V, I32, V, I32, ctypes.c_float,
                                           V, V, V, ctypes.c_size_t, V]
    assert lib.compressed_attn_decode(None, 1, 32, good, cache, None, 0, None, 10, None, 128, 0.1,
                                      None, None, None, 0, None) == 2                      # H = 32 at d = 512
    assert lib.compressed_attn_decode(None, 1, 64, good, cache, None, 0, None, 10, None, 128, 0.1,
                                      None, None, None, 0, None) == 1
    lib.compressed_attn_decode_workspace_size.argtypes = [I32, I32, Layout, I32, I32]
    lib.compressed_attn_decode_workspace_size.restype = ctypes.c_size_t
    assert lib.compressed_attn_decode_workspace_size(0, 64, good, 10, 128) == 0


def test_fused_selection_and_budget_host_paths(lib):
    """The fused decode selection validates like its two parts; the launch budget is
    a plain process-wide value (no device access on these paths)."""
    V, I32, I64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
    lib.lightning_index_topk.argtypes = [V, V, V, V, V, V, I32, I64, I32, I32, I32, I32, V, V, V, V,
                                         ctypes.c_size_t, V, V]
    P = V(0x1000)
    # unsupported c, Hi, k
    assert lib.lightning_index_topk(P, P, P, P, P, P, 2, 100, 4, 96, 4, 8, P, P, P, None, 0, None, None) == 2
    assert lib.lightning_index_topk(P, P, P, P, P, P, 2, 100, 9, 128, 4, 8, P, P, P, None, 0, None, None) == 2
    assert lib.lightning_index_topk(P, P, P, P, P, P, 2, 100, 4, 128, 4, 0, P, P, P, None, 0, None, None) == 2
    # bad m, null and misaligned pointers
    assert lib.lightning_index_topk(P, P, P, P, P, P, 2, 100, 4, 128, 0, 8, P, P, P, None, 0, None, None) == 1
    assert lib.lightning_index_topk(P, P, P, P, P, None, 2, 100, 4, 128, 4, 8, P, P, P, None, 0, None, None) == 1
    assert lib.lightning_index_topk(P, P, P, V(0x1004), P, P, 2, 100, 4, 128, 4, 8, P, P, P, None, 0, None,
                                    None) == 1
    # a row longer than 2^19 scores needs the workspace
    assert lib.lightning_index_topk(P, P, P, P, P, P, 2, 1 << 20, 4, 128, 4, 8, P, P, P, None, 0, None,
                                    None) == 4
    # no sequences: nothing to do
    assert lib.lightning_index_topk(None, None, None, None, None, None, 0, 100, 4, 128, 4, 8, None, None, None,
                                    None, 0, None, None) == 0
    lib.lightning_index_topk_workspace_size.argtypes = [I32, I64, I32]
    lib.lightning_index_topk_workspace_size.restype = ctypes.c_size_t
    lib.topk_select_workspace_size.argtypes = [I32, I64, I32]
    lib.topk_select_workspace_size.restype = ctypes.c_size_t
    assert lib.lightning_index_topk_workspace_size(4, 262144, 1024) == lib.topk_select_workspace_size(4, 262144, 1024)

    lib.hca_set_launch_budget.argtypes = [ctypes.c_int, ctypes.c_int]
    lib.hca_set_launch_budget.restype = ctypes.c_int
    prev = lib.hca_set_launch_budget(0, 60)
    assert prev >= 0
    assert lib.hca_set_launch_budget(0, prev) == 60
    assert lib.hca_set_launch_budget(1, 0) >= 0
    assert lib.hca_set_launch_budget(2, 10) == 0        # the decode indexer's budget
    assert lib.hca_set_launch_budget(2, 0) == 10
    assert lib.hca_set_launch_budget(3, 10) == -1       # unknown op
    assert lib.hca_set_launch_budget(0, -1) == -1       # negative budget
    lib.hca_set_early_query.argtypes = [ctypes.c_int]
    lib.hca_set_early_query.restype = ctypes.c_int
    prev = lib.hca_set_early_query(1)
    assert prev in (0, 1)
    assert lib.hca_set_early_query(prev) == 1
    assert lib.hca_set_early_query(2) == -1             # only 0 or 1
    assert lib.hca_set_early_query(-1) == -1


class EntryEx(ctypes.Structure):
    _fields_ = [("norm_w", ctypes.c_void_p), ("norm_eps", ctypes.c_float), ("inv_freq", ctypes.c_void_p)]


class AttnEx(ctypes.Structure):
    _fields_ = [("q_norm_w", ctypes.c_void_p), ("norm_eps", ctypes.c_float), ("sink", ctypes.c_void_p),
                ("inv_freq", ctypes.c_void_p), ("q_pos", ctypes.c_void_p), ("win_len", ctypes.c_void_p)]


def test_extension_calls_validate_on_the_host(lib):
    """The section 9 extras, the overlapped and key compressors, the BF16-score
    and 64-head indexer calls, the state-cache append and the host-to-host
    step reject bad arguments before any CUDA call."""
    V, I32, I64, F, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
    P, good = V(0x1000), Layout(512, 64, 64)
    cache = Cache(0x1000, 0x1000, 0x1000, 10)
    lib.csa_compress_ex.argtypes = [V, V, I64, V, I32, I64, Layout, Cache, I64, ctypes.POINTER(EntryEx), V]
    bad_w = EntryEx(0x1004, 1e-6, None)                                  # misaligned weight
    assert lib.csa_compress_ex(P, P, 8, P, 1, 1, good, cache, 0, ctypes.byref(bad_w), None) == 1
    neg = EntryEx(None, -1.0, None)                                      # negative epsilon
    assert lib.csa_compress_ex(P, P, 8, P, 1, 1, good, cache, 0, ctypes.byref(neg), None) == 1
    lib.kv_token_prep.argtypes = [V, V, I64, Layout, ctypes.POINTER(EntryEx), V, V]
    assert lib.kv_token_prep(P, P, 4, Layout(256, 64, 64), None, P, None) == 2
    assert lib.kv_token_prep(None, P, 4, good, None, P, None) == 1
    assert lib.kv_token_prep(None, None, 0, good, None, None, None) == 0
    lib.compressed_attn_decode_ex.argtypes = [V, I32, I32, Layout, Cache, V, I32, V, I32, V, I32, F,
                                              ctypes.POINTER(AttnEx), V, V, V, SZ, V]
    no_pos = AttnEx(None, 1e-6, None, 0x1000, None, None)                # RoPE without query positions
    assert lib.compressed_attn_decode_ex(P, 1, 64, good, cache, None, 0, P, 10, P, 128, 0.1, ctypes.byref(no_pos),
                                         P, None, None, 0, None) == 1
    lib.compressed_attn_prefill_ex.argtypes = [V, I32, I32, I32, I32, Layout, Cache, V, I32, V, V, I32, F,
                                               ctypes.POINTER(AttnEx), V, V]
    win_pf = AttnEx(None, 1e-6, None, None, None, 0x1000)                # window lengths are a decode input
    assert lib.compressed_attn_prefill_ex(P, 4, 64, 100, 4, good, cache, None, 0, None, P, 128, 0.1,
                                          ctypes.byref(win_pf), P, None) == 1
    lib.csa_compress_overlap.argtypes = [V, V, V, V, V, V, I64, V, I32, I64, Layout, Cache, I64, V]
    assert lib.csa_compress_overlap(P, P, P, P, P, None, 8, P, 1, 2, good, cache, 1, None) == 1    # a_prev alone
    assert lib.csa_compress_overlap(P, P, P, P, None, None, 7, P, 1, 2, good, cache, 0, None) == 1  # 8 rows needed
    lib.indexer_key_compress.argtypes = [V, V, V, V, V, V, I64, V, I32, I64, I32, V, V, I64, I64, V]
    assert lib.indexer_key_compress(P, P, P, P, None, None, 8, P, 1, 2, 96, P, P, 10, 0, None) == 2  # c = 96
    assert lib.indexer_key_compress(P, P, P, P, None, None, 8, P, 1, 2, 128, P, P, 1, 0, None) == 1  # capacity
    lib.lightning_index_ex.argtypes = [V, V, V, V, V, V, I32, I32, I64, I32, I32, I32, I32, V, V]
    assert lib.lightning_index_ex(P, P, P, P, P, P, 1, 1, 10, 4, 64, 4, 1, P, None) == 2     # BF16 needs c = 128
    assert lib.lightning_index_ex(P, P, P, P, P, P, 1, 1, 10, 64, 64, 4, 0, P, None) == 2    # 64 heads: c = 128
    assert lib.lightning_index_ex(P, P, P, P, P, P, 1, 1, 10, 16, 128, 4, 0, P, None) == 2   # 16 heads
    lib.topk_select_ex.argtypes = [V, I32, V, I32, I64, I32, I32, V, V, V, SZ, V]
    assert lib.topk_select_ex(P, 1, P, 2, 1000, 4, 8, P, P, None, 0, None) == 4              # BF16: workspace
    lib.topk_select_ex_workspace_size.argtypes = [I32, I64, I32, I32]
    lib.topk_select_ex_workspace_size.restype = SZ
    assert lib.topk_select_ex_workspace_size(2, 1000, 8, 1) > 0                               # any row length
    assert lib.topk_select_ex_workspace_size(2, 1000, 8, 0) == 0
    lib.kv_state_append.argtypes = [V, V, V, I32, I32, I64, V, I32, V, V, I32, V]
    assert lib.kv_state_append(P, P, None, 2, 100, 5, P, 128, P, P, 4, None) == 1            # d % 8 != 0
    assert lib.kv_state_append(P, P, None, 2, 128, -1, P, 128, P, P, 4, None) == 1           # negative position
    lib.hca_decode_step_host.argtypes = [V, V, V, V, V, V, V, V, V]
    assert lib.hca_decode_step_host(None, P, P, P, P, P, P, P, None) == 1


def test_step_host_packing_bits_checked_before_any_queue(lib):
    """hca_decode_step_host takes one copy for packed buffers only when the plan
    says so, and then checks the layout it states: a packing bit whose pointers
    do not lie that way (or an unknown bit) is refused before anything is
    queued, so this runs without a device."""
    from long_context_attention_hca_b200 import DecodeStepPlan, Layout
    V = ctypes.c_void_p
    lib.hca_decode_step_host.argtypes = [ctypes.POINTER(DecodeStepPlan), V, V, V, V, V, V, V, V]
    p = DecodeStepPlan()
    p.B, p.H, p.Hi, p.c, p.k, p.W = 4, 64, 4, 128, 1024, 128
    p.layout = Layout(512, 64, 64)
    p.side_stream = p.ev_fork = p.ev_index = p.ev_q = p.ev_join = p.ev_iq = 0x1000
    p.iq_codes, p.iq_sf, p.iq_w = 0x100000, 0x100400, 0x100440           # packed on the device
    p.out_csa, p.out_hca = 0x200000, 0x240000                             # packed on the device
    hq, hc, hs, hw = 0x300000, 0x400000, 0x500000, 0x600000               # host arrays apart
    ho_c, ho_h = 0x700000, 0x800000
    for bits in (1, 2, 4):
        p.packed = bits
        assert lib.hca_decode_step_host(ctypes.byref(p), hq, hq, hc, hs, hw, ho_c, ho_h, None) == 1, bits
