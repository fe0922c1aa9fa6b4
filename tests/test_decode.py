"""Split-K/V decode: one query row per head against N cached keys, checked
element by element against the fp64 oracle (attention_qk), same tolerances
as the forward pass."""
import math

import numpy as np
import pytest
import torch

import exact_attention_127_b200 as attn
import oracle
from exact_attention_127_b200 import inputs

O_MAX_ABS, O_REL_L2, LSE_MAX_ABS = 2e-2, 5e-3, 1e-3
FAKE = 0x10000


def test_decode_validation_on_host():
    lib = attn.load_library()
    ws = 1 << 20
    args = (FAKE, FAKE + 0x100000, FAKE + 0x200000, FAKE + 0x300000, FAKE + 0x400000)
    assert lib.attn_decode(*args, 1, 2, 100, 96, 0.1, FAKE + 0x500000, ws, None) == -3
    assert lib.attn_decode(*args, 1, 2, 100, 64, 0.0, FAKE + 0x500000, ws, None) == -5
    assert lib.attn_decode(*args, -1, 2, 100, 64, 0.1, FAKE + 0x500000, ws, None) == -4
    assert lib.attn_decode(None, *args[1:], 1, 2, 100, 64, 0.1, FAKE + 0x500000, ws, None) == -1
    assert lib.attn_decode(*args, 1, 2, 100, 64, 0.1, None, ws, None) == -11
    assert lib.attn_decode(*args, 1, 2, 100, 64, 0.1, FAKE + 0x500000, 8, None) == -11
    assert lib.attn_decode(*args, 0, 2, 100, 64, 0.1, None, 0, None) == 0
    assert lib.attn_decode_workspace_bytes(1, 2, 100, 80) == 0
    need = lib.attn_decode_workspace_bytes(16, 16, 8192, 128)
    assert need >= 16 * 16 * 128 * 4   # at least one fp32 partial per head
    # one partial per (head, CTA) pair that shares keys: at most B*H + 159 of them
    # (d fp32 values, 256-byte aligned, then an (m, l) pair each); independent of N
    for B, H, N, d in [(16, 16, 8192, 128), (1, 1, 1, 64), (32, 32, 4096, 64)]:
        slots = B * H + 159
        expect = (slots * d * 4 + 255) // 256 * 256 + slots * 8
        assert lib.attn_decode_workspace_bytes(B, H, N, d) == expect


@pytest.fixture(scope="module")
def gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    attn.load_library()
    assert attn.device_status(reset=True) == 0


def _check(q, k, v, label):
    B, H, N, d = k.shape
    o, lse = attn.attn_decode(q.cuda(), k.cuda(), v.cuda())
    torch.cuda.synchronize()
    assert attn.device_status(reset=True) == 0
    O, L = oracle.attention_qk(q, k, v, 1.0 / math.sqrt(d))
    of = o.cpu().reshape(B * H, 1, d).double().numpy()
    lf = lse.cpu().reshape(B * H, 1).double().numpy()
    err = np.abs(of - O).max()
    rel = np.linalg.norm(of - O) / np.linalg.norm(O)
    lerr = np.abs(lf - L).max()
    msg = f"{label}: max|dO|={err:.3e} relL2={rel:.3e} max|dLSE|={lerr:.3e}"
    assert err <= O_MAX_ABS and rel <= O_REL_L2 and lerr <= LSE_MAX_ABS, msg


@pytest.mark.gpu
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("N", [1, 2, 31, 32, 33, 127, 128, 129, 1000, 5000])
def test_decode_edge_lengths(gpu, N, d):
    q, k, v = inputs.make_decode_qkv(2, 3, N, d, seed=200 + N)
    _check(q, k, v, f"N={N} d={d}")


@pytest.mark.gpu
def test_decode_many_splits_single_head(gpu):
    # one head: the plan cuts the keys into many splits of 128-key multiples
    q, k, v = inputs.make_decode_qkv(1, 1, 70000, 128, seed=9)
    _check(q, k, v, "one head, 70000 keys")


@pytest.mark.gpu
def test_decode_peaked_scores(gpu):
    q, k, v = inputs.make_decode_qkv(2, 4, 3000, 128, seed=10)
    k[:, :, 1234] = (q[:, :, 0].float() * 8).to(torch.bfloat16)   # one dominant key
    _check(q, k, v, "peaked")


@pytest.mark.gpu
@pytest.mark.parametrize("name", sorted(inputs.DECODE_WORKLOADS))
def test_decode_workloads(gpu, name):
    w = inputs.DECODE_WORKLOADS[name]
    q, k, v = inputs.make_decode_qkv(w.B, w.H, w.N, w.d, w.seed)
    _check(q, k, v, name)


@pytest.mark.gpu
def test_decode_deterministic_and_shapes(gpu):
    q, k, v = (t.cuda() for t in inputs.make_decode_qkv(2, 2, 4097, 64, seed=11))
    o1, l1 = attn.attn_decode(q, k, v)
    o2, l2 = attn.attn_decode(q[:, :, 0].contiguous(), k, v)
    torch.cuda.synchronize()
    assert o1.shape == (2, 2, 1, 64) and o2.shape == (2, 2, 64) and l1.shape == (2, 2)
    assert torch.equal(o1[:, :, 0], o2) and torch.equal(l1, l2)
