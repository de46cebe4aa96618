"""Seeded synthetic inputs for the CSA/HCA hot path.

This module is the only code shared by the oracle side (tests) and the GPU
side (tests, bench, smoke).  It holds shapes and random-number draws and none
of the method's arithmetic.

Workloads (the five synthetic configurations the path is checked and timed
on; value distributions are those of the "DeepSeek V4 ..." reading note's
parameters, section 7: m = 4, indexer head dim 128, window 128, top-k 512 /
1024; section 8: m' = 128):

  tiny_decode_1k     B=1,  t=1023,      d=128 (96 FP8 + 32 bf16 rope), g=32, H=8,
                     indexer 4 x 64, k=32                          (seed 0)
  decode_b16_64k     B=16, t=65535,     d=512 (448 + 64), g=64, H=64,
                     indexer 4 x 128, k=512                        (seed 1)
  decode_b4_1m       B=4,  t=1048575,   same dims, k=1024           (seed 2)
  prefill_4096_131k  B=1, 4096 queries at 131072..135167 after 131072
                     compressed tokens, k=1024                      (seed 3)
  stack61_b32_256k   B=32, t=262143, 61 layers (30 CSA + 31 HCA), k=1024 (seed 4)

Draws:  raw KV x and gate logits ~ N(0, 1) rounded to bf16; positional bias
~ N(0, 0.5) fp32 (0.5 read as the standard deviation); attention queries
~ N(0, 1) bf16; indexer query/key FP4 codes uniform over the 16 e2m1 codes
(a uniform byte holds two uniform nibbles); ue8m0 scales uniform over
123..127 (2^-4 .. 2^0); indexer head weights w ~ U(0, 1) fp32.

Each tensor has its own torch.Generator seeded from (workload seed, tensor
name, layer), so any tensor can be regenerated alone.  Values depend on the
device the generator runs on (torch's CPU and CUDA generators differ); the
oracle always receives host copies of exactly the tensors it checks.
"""
from __future__ import annotations

import dataclasses
import hashlib

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    seed: int
    B: int                 # sequences
    t: int                 # decode: query position; prefill: first query position
    d: int                 # channels per KV entry
    d_rope: int            # trailing channels kept bf16
    g: int                 # FP8 scale group (channels)
    H: int                 # attention query heads
    Hi: int                # indexer heads
    c: int                 # indexer head dim
    k: int                 # top-k
    W: int = 128           # sliding window
    m_csa: int = 4
    m_hca: int = 128
    Tq: int = 1            # queries per sequence (prefill chunk length)
    layers: int = 1        # attention layers (stack workload)

    @property
    def prefill(self) -> bool:
        return self.Tq > 1

    @property
    def n_tokens(self) -> int:
        """Raw tokens in each sequence (context incl. the query tokens)."""
        return self.t + self.Tq

    @property
    def softmax_scale(self) -> float:
        return float(self.d) ** -0.5


WORKLOADS = {
    "tiny_decode_1k": Workload("tiny_decode_1k", 0, B=1, t=1023, d=128, d_rope=32, g=32, H=8, Hi=4, c=64, k=32),
    "decode_b16_64k": Workload("decode_b16_64k", 1, B=16, t=65535, d=512, d_rope=64, g=64, H=64, Hi=4, c=128, k=512),
    "decode_b4_1m": Workload("decode_b4_1m", 2, B=4, t=1048575, d=512, d_rope=64, g=64, H=64, Hi=4, c=128, k=1024),
    "prefill_4096_131k": Workload("prefill_4096_131k", 3, B=1, t=131072, d=512, d_rope=64, g=64, H=64, Hi=4, c=128,
                                  k=1024, Tq=4096),
    "stack61_b32_256k": Workload("stack61_b32_256k", 4, B=32, t=262143, d=512, d_rope=64, g=64, H=64, Hi=4, c=128,
                                 k=1024, layers=61),
}


def _seed(wl_seed: int, name: str, layer: int) -> int:
    h = hashlib.sha256(f"{wl_seed}/{name}/{layer}".encode()).digest()
    return int.from_bytes(h[:8], "little") & ((1 << 63) - 1)


def generator(wl_seed: int, name: str, layer: int = 0, device="cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(_seed(wl_seed, name, layer))
    return g


def normal_bf16(shape, std, wl_seed, name, layer=0, device="cpu") -> torch.Tensor:
    g = generator(wl_seed, name, layer, device)
    return (torch.randn(shape, generator=g, device=device, dtype=torch.float32) * std).to(torch.bfloat16)


def normal_f32(shape, std, wl_seed, name, layer=0, device="cpu") -> torch.Tensor:
    g = generator(wl_seed, name, layer, device)
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32) * std


def uniform_bytes(shape, wl_seed, name, layer=0, device="cpu") -> torch.Tensor:
    g = generator(wl_seed, name, layer, device)
    return torch.randint(0, 256, shape, generator=g, device=device, dtype=torch.uint8)


def ue8m0_scales(shape, wl_seed, name, layer=0, device="cpu", lo=123, hi=127) -> torch.Tensor:
    g = generator(wl_seed, name, layer, device)
    return torch.randint(lo, hi + 1, shape, generator=g, device=device, dtype=torch.uint8)


def uniform_f32(shape, wl_seed, name, layer=0, device="cpu") -> torch.Tensor:
    g = generator(wl_seed, name, layer, device)
    return torch.rand(shape, generator=g, device=device, dtype=torch.float32)


def bf16_bits(t: torch.Tensor):
    """bf16 tensor -> numpy uint16 bit patterns (host copy)."""
    return t.detach().to("cpu").contiguous().view(torch.int16).numpy().view("uint16")


# ------------------------------------------------------------------ per-tensor recipes
def raw_kv(wl: Workload, B, T, layer=0, device="cpu", t0=0):
    """x, gate: [B][T][d] bf16 for tokens t0..t0+T-1 (token rows are drawn
    from one stream per sequence so a slice is reproducible only from t0=0;
    callers that need a slice generate the whole sequence)."""
    assert t0 == 0
    x = normal_bf16((B, T, wl.d), 1.0, wl.seed, "x", layer, device)
    gate = normal_bf16((B, T, wl.d), 1.0, wl.seed, "gate", layer, device)
    return x, gate


def pos_bias(wl: Workload, m: int, layer=0, device="cpu"):
    return normal_f32((m, wl.d), 0.5, wl.seed, f"bias{m}", layer, device)


def queries(wl: Workload, rows: int, layer=0, device="cpu"):
    """Attention queries [rows][H][d] bf16."""
    return normal_bf16((rows, wl.H, wl.d), 1.0, wl.seed, "q", layer, device)


def indexer_queries(wl: Workload, rows: int, layer=0, device="cpu"):
    """(codes [rows][Hi][c/2], ue8m0 [rows][Hi][c/32], w [rows][Hi])."""
    qc = uniform_bytes((rows, wl.Hi, wl.c // 2), wl.seed, "iq", layer, device)
    qs = ue8m0_scales((rows, wl.Hi, wl.c // 32), wl.seed, "iqs", layer, device)
    w = uniform_f32((rows, wl.Hi), wl.seed, "iw", layer, device)
    return qc, qs, w


def indexer_keys(wl: Workload, B: int, n: int, layer=0, device="cpu"):
    """(codes [B][n][c/2], ue8m0 [B][n][c/32])."""
    kc = uniform_bytes((B, n, wl.c // 2), wl.seed, "ik", layer, device)
    ks = ue8m0_scales((B, n, wl.c // 32), wl.seed, "iks", layer, device)
    return kc, ks


# ------------------------------------------------------------------ section 9 extras (parameters, not arithmetic)
NORM_EPS = 1e-6
ROPE_BASE = 10000.0


def rope_inv_freq(d_rope: int, base: float = ROPE_BASE, device="cpu"):
    """RoPE frequency table fp32 [d_rope/2]: base^(-2i/d_rope), rounded to fp32
    (the usual rotary table; the pages fix no base)."""
    import numpy as np
    f = (base ** (-np.arange(0, d_rope, 2, dtype=np.float64) / d_rope)).astype(np.float32)
    return torch.from_numpy(f).to(device)


def section9_params(wl: Workload, layer=0, device="cpu"):
    """Learned-parameter stand-ins for the note's section 9 extras: KV-entry
    and query RMSNorm weights ~ 1 + N(0, 0.1) fp32 [d], per-head sink logits
    ~ N(0, 1) fp32 [H], and the RoPE table."""
    kvw = 1.0 + normal_f32((wl.d,), 0.1, wl.seed, "kv_norm_w", layer, device)
    qw = 1.0 + normal_f32((wl.d,), 0.1, wl.seed, "q_norm_w", layer, device)
    sink = normal_f32((wl.H,), 1.0, wl.seed, "sink", layer, device)
    return {"kv_norm_w": kvw, "q_norm_w": qw, "sink": sink, "inv_freq": rope_inv_freq(wl.d_rope, device=device),
            "eps": NORM_EPS}

