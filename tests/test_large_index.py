"""Element offsets beyond 2^31: the forward (bf16 and e4m3), backward and
decode entry points on tensors of more than 2^31 elements.

B=1, H=8200, N=2048, d=128 makes 2.15e9 elements per [B, H, N, d] tensor, so
the last heads' elements lie past the range of a 32-bit index (the bf16
tensors are 4.3 GB each; the backward holds about 43 GB in all).  Two heads,
the first and the last, carry seeded data and are checked against the fp64
oracle; the other heads are zero, which fixes their outputs in closed form
(all scores 0: O = mean of zero values = 0, LSE = ln of the number of allowed
keys; with dO = 0 every gradient is 0).
"""
import math

import numpy as np
import pytest
import torch

import exact_attention_127_b200 as attn
import oracle
from exact_attention_127_b200 import inputs

pytestmark = pytest.mark.gpu

B, H, N, D = 1, 8200, 2048, 128
FILLED = (0, H - 1)
MID = H // 2
SCALE = 1.0 / math.sqrt(D)
O_MAX_ABS, O_REL_L2, LSE_MAX_ABS = 2e-2, 5e-3, 1e-3


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    assert B * H * N * D > 2**31
    free, _ = torch.cuda.mem_get_info()
    if free < 60 * 2**30:
        pytest.skip("needs about 60 GB of free device memory")
    attn.load_library()
    assert attn.device_status(reset=True) == 0
    return attn


def _big(fill):
    """Zero [B, H, N, D] bf16 device tensor with `fill` ([2, N, D], CPU) in the FILLED heads."""
    t = torch.zeros((B, H, N, D), dtype=torch.bfloat16, device="cuda")
    for j, h in enumerate(FILLED):
        t[0, h].copy_(fill[j])
    return t


def _release():
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


def test_forward_beyond_2_31_elements(lib):
    sq, sk, sv = (t[0] for t in inputs.make_qkv(1, 2, N, D, seed=61))
    q, k, v = _big(sq), _big(sk), _big(sv)
    o, lse = lib.attn_fwd(q, k, v, causal=True, scale=SCALE)
    torch.cuda.synchronize()
    assert lib.device_status(reset=True) == 0
    rows = inputs.sample_rows(N, 128, 61)
    O_ref, L_ref = oracle.attention_rows(sq[None], sk[None], sv[None], True, SCALE, rows=rows)
    of = o[0, list(FILLED)][:, rows].double().cpu().numpy()
    lf = lse[0, list(FILLED)][:, rows].double().cpu().numpy()
    err = np.abs(of - O_ref)
    rel = np.linalg.norm(of - O_ref) / np.linalg.norm(O_ref)
    assert err.max() <= O_MAX_ABS and rel <= O_REL_L2, (err.max(), rel)
    assert np.abs(lf - L_ref).max() <= LSE_MAX_ABS
    # a zero head: O = 0 exactly, LSE_i = ln(i + 1)
    assert not o[0, MID].any()
    want = torch.log(torch.arange(1, N + 1, dtype=torch.float64))
    assert (lse[0, MID].double().cpu() - want).abs().max().item() <= 1e-4
    del q, k, v, o, lse
    _release()


def test_backward_beyond_2_31_elements(lib):
    sq, sk, sv = (t[0] for t in inputs.make_qkv(1, 2, N, D, seed=62))
    sdo = inputs.make_qkv(1, 2, N, D, seed=63)[0][0]
    q, k, v, dout = _big(sq), _big(sk), _big(sv), _big(sdo)
    o, lse = lib.attn_fwd(q, k, v, causal=True, scale=SCALE)
    dq, dk, dv = lib.attn_bwd(q, k, v, o, lse, dout, causal=True, scale=SCALE)
    torch.cuda.synchronize()
    assert lib.device_status(reset=True) == 0
    ref = oracle.attention_backward(sq[None], sk[None], sv[None], sdo[None], True, SCALE)
    for name, g, r in zip(("dq", "dk", "dv"), (dq, dk, dv), ref):
        gf = g[0, list(FILLED)].double().cpu().numpy()
        rel = np.linalg.norm(gf - r) / np.linalg.norm(r)
        err = np.abs(gf - r).max()
        assert rel <= 1e-2 and err <= 3e-2 * np.abs(r).max() + 1e-3, (name, rel, err)
        assert not g[0, MID].any(), name            # dO = 0 there: every gradient is 0
    del q, k, v, dout, o, lse, dq, dk, dv
    _release()


def test_decode_beyond_2_31_elements(lib):
    sq, sk, sv = (t[0] for t in inputs.make_decode_qkv(1, 2, N, D, seed=64))
    q = torch.zeros((B, H, 1, D), dtype=torch.bfloat16, device="cuda")
    for j, h in enumerate(FILLED):
        q[0, h].copy_(sq[j])
    k, v = _big(sk), _big(sv)
    o, lse = lib.attn_decode(q, k, v, scale=SCALE)
    torch.cuda.synchronize()
    assert lib.device_status(reset=True) == 0
    O_ref, L_ref = oracle.attention_qk(sq[None], sk[None], sv[None], SCALE)
    of = o[0, list(FILLED)].double().cpu().numpy()
    lf = lse[0, list(FILLED)].double().cpu().numpy()
    assert np.abs(of - O_ref).max() <= O_MAX_ABS
    assert np.abs(lf.reshape(L_ref.shape) - L_ref).max() <= LSE_MAX_ABS
    # a zero head: O = 0, LSE = ln N
    assert not o[0, MID].any()
    assert abs(lse[0, MID].item() - math.log(N)) <= 1e-4
    del q, k, v, o, lse
    _release()


def test_fp8_forward_beyond_2_31_elements(lib):
    """e4m3 operands (1 byte per element, so 2.15 GB per tensor, and V^T in the
    workspace), checked like tests/test_fp8.py: the oracle on the dequantized
    values, per-element bound (2^-4 + 2^-8) max_j |v_jc| + 1e-3, relative L2
    below 5 %."""
    sq, sk, sv = (t[0] for t in inputs.make_qkv_e4m3(1, 2, N, D, seed=65))

    def big8(fill):
        t = torch.zeros((B, H, N, D), dtype=torch.float8_e4m3fn, device="cuda")
        for j, h in enumerate(FILLED):
            t[0, h].copy_(fill[j])
        return t

    q8, k8, v8 = big8(sq), big8(sk), big8(sv)
    o, lse = lib.attn_fwd_fp8(q8, k8, v8, causal=True, scale=SCALE)
    torch.cuda.synchronize()
    assert lib.device_status(reset=True) == 0
    rows = inputs.sample_rows(N, 128, 65)
    qd, kd, vd = (t.to(torch.float64)[None] for t in (sq, sk, sv))
    O_ref, L_ref = oracle.attention_rows(qd, kd, vd, True, SCALE, rows=rows)
    of = o[0, list(FILLED)][:, rows].double().cpu().numpy()
    lf = lse[0, list(FILLED)][:, rows].double().cpu().numpy()
    vmax = np.maximum.accumulate(np.abs(vd[0].numpy()), axis=1)[:, rows]     # over keys j <= i
    assert np.all(np.abs(of - O_ref) <= (2.0 ** -4 + 2.0 ** -8) * vmax + 1e-3)
    assert np.linalg.norm(of - O_ref) / np.linalg.norm(O_ref) <= 5e-2
    assert np.abs(lf - L_ref).max() <= LSE_MAX_ABS
    assert not o[0, MID].any()
    del q8, k8, v8, o, lse
    _release()

