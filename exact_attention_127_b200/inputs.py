"""Seeded synthetic inputs shared by the tests, the smoke check and the bench.

This module holds random-number recipes and shapes only -- none of the
attention arithmetic -- so that the CUDA path and the CPU oracle can be fed the
very same bf16 bytes without sharing any computation.

Recipe (the same for every workload): a CPU ``torch.Generator`` seeded with the
workload's seed draws fp32 samples for Q, then K, then V, each of shape
[B, H, N, d] in that order; each tensor is then rounded to bf16
(round-to-nearest-even).  The standard workload draws all three from N(0, 1).
The large-logit workload draws Q and K from N(0, 4^2) and V from U(-1, 1).
"""
from __future__ import annotations

import hashlib
import math
from dataclasses import dataclass

import numpy as np
import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    d: int
    causal: bool
    seed: int
    qk_std: float = 1.0
    v_dist: str = "normal"     # "normal" (N(0,1)) or "uniform" (U(-1,1))
    note: str = ""

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def shape(self):
        return (self.B, self.H, self.N, self.d)

    def flops(self) -> float:
        """Useful forward FLOPs: 4*B*H*N^2*d, halved when causal."""
        f = 4.0 * self.B * self.H * self.N * self.N * self.d
        return f / 2.0 if self.causal else f

    def compulsory_bytes(self) -> int:
        """Q, K, V read and O written once (bf16) plus LSE written once (fp32)."""
        return 2 * 4 * self.B * self.H * self.N * self.d + 4 * self.B * self.H * self.N


# The five workloads: a tiny single-tile case, prefill-like medium and long
# sequences, a long-context large-logit case and a short-sequence many-heads case.
WORKLOADS = {
    "tiny_n128_d64": Workload("tiny_n128_d64", 1, 1, 128, 64, False, 0,
                              note="single 128-row tile"),
    "b8h16_n2048_d64": Workload("b8h16_n2048_d64", 8, 16, 2048, 64, False, 1),
    "b4h16_n8192_d128_causal": Workload("b4h16_n8192_d128_causal", 4, 16, 8192, 128, True, 2,
                                        note="headline workload"),
    "b1h16_n32768_d128_causal_peaked": Workload(
        "b1h16_n32768_d128_causal_peaked", 1, 16, 32768, 128, True, 3, qk_std=4.0,
        v_dist="uniform", note="Q,K ~ N(0,16), V ~ U(-1,1): large, peaked logits"),
    "b32h32_n512_d64": Workload("b32h32_n512_d64", 32, 32, 512, 64, False, 4,
                                note="short sequences, many heads"),
}
WORKLOAD_ORDER = list(WORKLOADS)
HEADLINE = "b4h16_n8192_d128_causal"


def make_qkv(B: int, H: int, N: int, d: int, seed: int, qk_std: float = 1.0,
             v_dist: str = "normal"):
    """Seeded bf16 CPU tensors q, k, v of shape [B, H, N, d]."""
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    shape = (B, H, N, d)
    q = torch.randn(shape, generator=g, dtype=torch.float32)
    k = torch.randn(shape, generator=g, dtype=torch.float32)
    if qk_std != 1.0:
        q.mul_(qk_std)
        k.mul_(qk_std)
    if v_dist == "normal":
        v = torch.randn(shape, generator=g, dtype=torch.float32)
    elif v_dist == "uniform":
        v = torch.rand(shape, generator=g, dtype=torch.float32).mul_(2.0).sub_(1.0)
    else:
        raise ValueError(f"unknown v_dist {v_dist!r}")
    return q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16)


def make_qkv_e4m3(B: int, H: int, N: int, d: int, seed: int, amplitude: float = 1.0,
                  descale: float = 1.0):
    """Seeded e4m3 (torch.float8_e4m3fn) CPU tensors for the 8-bit forward:
    make_qkv's bf16 draws times `amplitude`, divided by `descale` and rounded
    to e4m3 (nearest even).  The attention they stand for is that of
    x8 * descale, which is exact in fp64."""
    out = []
    for t in make_qkv(B, H, N, d, seed):
        x = t.float() * float(amplitude) / float(descale)
        out.append(x.to(torch.float8_e4m3fn))
    return tuple(out)


@dataclass(frozen=True)
class DecodeWorkload:
    """One new query row per head against N cached keys (decode)."""
    name: str
    B: int
    H: int
    N: int
    d: int
    seed: int

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    def flops(self) -> float:
        return 4.0 * self.B * self.H * self.N * self.d

    def compulsory_bytes(self) -> int:
        """K and V read once (the cache), q read and o written (bf16), lse written."""
        return 2 * 2 * self.B * self.H * self.N * self.d + 2 * 2 * self.B * self.H * self.d \
            + 4 * self.B * self.H


DECODE_WORKLOADS = {
    "decode_b16h16_n8192_d128": DecodeWorkload("decode_b16h16_n8192_d128", 16, 16, 8192, 128, 5),
    "decode_b4h16_n32768_d128": DecodeWorkload("decode_b4h16_n32768_d128", 4, 16, 32768, 128, 6),
    "decode_b32h32_n4096_d64": DecodeWorkload("decode_b32h32_n4096_d64", 32, 32, 4096, 64, 7),
}


def make_decode_qkv(B: int, H: int, N: int, d: int, seed: int):
    """Seeded bf16 CPU tensors: q [B, H, 1, d] drawn first, then k and v
    [B, H, N, d], all N(0, 1), each rounded to bf16 (RNE)."""
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    q = torch.randn((B, H, 1, d), generator=g, dtype=torch.float32)
    k = torch.randn((B, H, N, d), generator=g, dtype=torch.float32)
    v = torch.randn((B, H, N, d), generator=g, dtype=torch.float32)
    return q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16)


def workload_inputs(w: Workload):
    return make_qkv(w.B, w.H, w.N, w.d, w.seed, w.qk_std, w.v_dist)


def digest(*tensors) -> str:
    """SHA-256 over the raw bytes of the given CPU tensors (input identity)."""
    h = hashlib.sha256()
    for t in tensors:
        h.update(t.contiguous().view(torch.uint8).numpy().tobytes())
    return h.hexdigest()


def sample_rows(N: int, count: int, seed: int) -> np.ndarray:
    """Seeded sample of query rows: tile- and diagonal-boundary rows
    {0, 1, 127, 128, 129, N-129, N-128, N-1} plus uniform draws without
    replacement from numpy's default_rng(1000 + seed), sorted."""
    fixed = {r for r in (0, 1, 127, 128, 129, N - 129, N - 128, N - 1) if 0 <= r < N}
    if count >= N:
        return np.arange(N, dtype=np.int64)
    rng = np.random.default_rng(1000 + int(seed))
    rest = [r for r in rng.permutation(N).tolist() if r not in fixed]
    rows = sorted(fixed | set(rest[:max(0, count - len(fixed))]))
    return np.asarray(rows, dtype=np.int64)
