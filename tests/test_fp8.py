"""The forward pass on e4m3 inputs (attn_fwd_fp8) against the fp64 oracle.

The oracle is the plain definition evaluated on the dequantized inputs
(x8 * descale, exact in fp64), so the e4m3 rounding of q, k and v is not an
error here: it is the input.  The kernel's one extra rounding is P -> e4m3
before P V (3 mantissa bits, nearest even: relative error at most 2^-4 per
element).  With O_i = sum_j w_j v_j and w_j = p_j / l >= 0 summing to one, the
rounded weights give |dO_ic| <= 2^-4 * sum_j w_j |v_jc| <= 2^-4 * max_j |v_jc|,
and bf16 output rounding adds at most 2^-9 |O_ic| <= 2^-9 max_j |v_jc|.  The
per-element bound below is (2^-4 + 2^-8) max_j |v_jc| + 1e-3.  For independent
rounding errors the relative L2 error of O is about the rms relative error of
one rounding: at most 2^-4 / sqrt(3) = 3.6 % (values at the bottom of a binade,
where the relative spacing is 2^-3), about 2.5 % averaged over a binade.  The
suite allows 5 %.  The statistics stay
fp32 (l is summed before P is rounded), so LSE keeps the bf16 path's 1e-3.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from exact_attention_127_b200 import inputs

P_ROUND = 2.0 ** -4
O_REL_L2 = 5e-2
LSE_MAX_ABS = 1e-3
ATTN_ERR_HEADDIM, ATTN_ERR_SCALE, ATTN_ERR_WORKSPACE = -3, -5, -11


def _deq(x8, descale):
    return x8.to(torch.float64) * float(descale)


def _elem_bound(v, heads, rows, causal):
    """(2^-4 + 2^-8) * max over the row's allowed keys of |v_jc| + 1e-3."""
    vv = np.abs(v.reshape(-1, v.shape[2], v.shape[3])[heads])       # [h, N, d]
    if causal:
        cm = np.maximum.accumulate(vv, axis=1)[:, rows]             # max over keys j <= i
    else:
        cm = np.broadcast_to(vv.max(axis=1, keepdims=True), (len(heads), len(rows), vv.shape[2]))
    return (P_ROUND + 2.0 ** -8) * cm + 1e-3


def _check(o, lse, q, k, v, causal, scale, heads, rows, label):
    O_ref, L_ref = oracle.attention_rows(q, k, v, causal, scale, rows=rows, heads=heads)
    B, H, N, d = o.shape
    of = o.reshape(B * H, N, d)[heads][:, rows].double().numpy()
    lf = lse.reshape(B * H, N)[heads][:, rows].double().numpy()
    assert np.all(np.isfinite(of)) and np.all(np.isfinite(lf)), label
    err = np.abs(of - O_ref)
    bound = _elem_bound(v.numpy(), heads, rows, causal)
    rel = np.linalg.norm(of - O_ref) / max(np.linalg.norm(O_ref), 1e-30)
    lerr = np.abs(lf - L_ref).max()
    msg = (f"{label}: max|dO|/bound={(err / bound).max():.3f} relL2={rel:.3e} "
           f"max|dLSE|={lerr:.3e}")
    assert np.all(err <= bound), msg
    assert rel <= O_REL_L2, msg
    assert lerr <= LSE_MAX_ABS, msg
    return rel


# ---------------------------------------------------------------------------
# CPU: the error model behind the tolerances, on plain torch arithmetic
# ---------------------------------------------------------------------------
def test_e4m3_rounding_model_meets_the_bounds():
    """Rounding the softmax weights to e4m3 (torch's conversion, nearest even)
    and renormalising by the unrounded sum: the per-element bound holds and the
    relative L2 error lies below the 2^-4/sqrt(3) estimate, near 2.5 %."""
    g = torch.Generator().manual_seed(7)
    N, d = 2048, 128
    s = torch.randn(64, N, generator=g, dtype=torch.float64) * 2.0
    v = torch.randn(N, d, generator=g, dtype=torch.float64)
    m = s.max(dim=1, keepdim=True).values
    p = torch.exp2((s - m) * math.log2(math.e))
    l = p.sum(dim=1, keepdim=True)
    o = (p / l) @ v
    p8 = p.to(torch.float8_e4m3fn).to(torch.float64)
    o8 = (p8 / l) @ v
    err = (o8 - o).abs()
    assert torch.all(err <= P_ROUND * v.abs().max(dim=0).values + 1e-12)
    rel = (torch.linalg.norm(o8 - o) / torch.linalg.norm(o)).item()
    assert 0.015 < rel < P_ROUND / math.sqrt(3), rel


def test_binding_rejects_wrong_inputs():
    import exact_attention_127_b200 as m
    q = torch.zeros(1, 1, 4, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        m.attn_fwd_fp8(q, q, q)
    q8 = q.to(torch.float8_e4m3fn)
    with pytest.raises(ValueError):          # CPU tensors
        m.attn_fwd_fp8(q8, q8, q8)
    assert m.fp8_workspace_bytes(1, 1, 4, 96) == 0
    assert m.fp8_workspace_bytes(2, 3, 300, 128) == 2 * 3 * 128 * 384
    assert m.fp8_workspace_bytes(2, 3, 300, 64) == 2 * 3 * 64 * 384     # V^T [BH][d][Np]


# ---------------------------------------------------------------------------
# GPU parity
# ---------------------------------------------------------------------------
@pytest.fixture(scope="module")
def attn():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import exact_attention_127_b200 as m
    m.load_library()
    assert m.device_status(reset=True) == 0
    return m


def _run(attn, q8, k8, v8, ds, causal, scale):
    o, lse = attn.attn_fwd_fp8(q8.cuda(), k8.cuda(), v8.cuda(), ds[0], ds[1], ds[2],
                               causal=causal, scale=scale)
    torch.cuda.synchronize()
    assert attn.device_status(reset=True) == 0
    return o.cpu(), lse.cpu()


EDGE_N = [1, 2, 127, 128, 129, 255, 256, 257, 300, 385, 1000]


@pytest.mark.gpu
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", EDGE_N)
def test_edge_shapes(attn, N, causal, d):
    q8, k8, v8 = inputs.make_qkv_e4m3(1, 2, N, d, seed=300 + N)
    scale = 1.0 / math.sqrt(d)
    o, lse = _run(attn, q8, k8, v8, (1.0, 1.0, 1.0), causal, scale)
    q, k, v = (_deq(t, 1.0) for t in (q8, k8, v8))
    _check(o, lse, q, k, v, causal, scale, [0, 1], np.arange(N), f"N={N} causal={causal} d={d}")


@pytest.mark.gpu
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_descales(attn, causal, d):
    """Inputs with amplitude 40 (beyond e4m3's 448 after q.k growth is fine, but
    the values themselves need the descale): q8 = x / 4, k8 = x / 8, v8 = x / 16."""
    N = 700
    ds = (4.0, 8.0, 16.0)
    q8, _, _ = inputs.make_qkv_e4m3(1, 3, N, d, seed=41, amplitude=40.0, descale=ds[0])
    _, k8, _ = inputs.make_qkv_e4m3(1, 3, N, d, seed=41, amplitude=40.0, descale=ds[1])
    _, _, v8 = inputs.make_qkv_e4m3(1, 3, N, d, seed=41, amplitude=40.0, descale=ds[2])
    scale = 1.0 / (40.0 * 40.0 * math.sqrt(d))     # keeps the logits O(1)
    o, lse = _run(attn, q8, k8, v8, ds, causal, scale)
    q, k, v = _deq(q8, ds[0]), _deq(k8, ds[1]), _deq(v8, ds[2])
    _check(o, lse, q, k, v, causal, scale, [0, 1, 2], np.arange(N), f"descales causal={causal}")


@pytest.mark.gpu
def test_many_heads_more_units_than_sms(attn):
    q8, k8, v8 = inputs.make_qkv_e4m3(2, 40, 512, 128, seed=77)
    scale = 1.0 / math.sqrt(128)
    o, lse = _run(attn, q8, k8, v8, (1.0, 1.0, 1.0), True, scale)
    q, k, v = (_deq(t, 1.0) for t in (q8, k8, v8))
    heads = [0, 17, 41, 79]
    _check(o, lse, q, k, v, True, scale, heads, np.arange(512), "80 heads")


@pytest.mark.gpu
@pytest.mark.parametrize("name", ["b4h16_n8192_d128_causal", "b1h16_n32768_d128_causal_peaked",
                                  "b8h16_n2048_d64", "b32h32_n512_d64"])
def test_workload_sampled_rows(attn, name):
    """Full-size workloads (d = 128 and d = 64), in the launch configuration
    bench.py times, checked on sampled rows of sampled heads."""
    w = inputs.WORKLOADS[name]
    q8, k8, v8 = inputs.make_qkv_e4m3(w.B, w.H, w.N, w.d, seed=w.seed)
    o, lse = _run(attn, q8, k8, v8, (1.0, 1.0, 1.0), w.causal, w.scale)
    q, k, v = (_deq(t, 1.0) for t in (q8, k8, v8))
    BH = w.B * w.H
    heads = sorted({0, BH // 2, BH - 1})
    rows = inputs.sample_rows(w.N, 96, w.seed)
    _check(o, lse, q, k, v, w.causal, w.scale, heads, rows, name)


@pytest.mark.gpu
@pytest.mark.parametrize("d", [64, 128])
def test_close_to_the_bf16_kernel_on_the_same_values(attn, d):
    """e4m3 values are exact in bf16: the bf16 kernel sees the same inputs, and
    the two outputs differ only by the rounding of P (bf16 vs e4m3)."""
    N = 1024
    q8, k8, v8 = inputs.make_qkv_e4m3(1, 4, N, d, seed=9)
    scale = 1.0 / math.sqrt(d)
    o8, l8 = _run(attn, q8, k8, v8, (1.0, 1.0, 1.0), True, scale)
    qb, kb, vb = (t.to(torch.bfloat16).cuda() for t in (q8, k8, v8))
    ob, lb = attn.attn_fwd(qb, kb, vb, causal=True, scale=scale)
    torch.cuda.synchronize()
    ob, lb = ob.cpu().double(), lb.cpu().double()
    rel = (torch.linalg.norm(o8.double() - ob) / torch.linalg.norm(ob)).item()
    assert rel < O_REL_L2, rel
    assert (l8.double() - lb).abs().max().item() < 2 * LSE_MAX_ABS


@pytest.mark.gpu
def test_error_codes(attn):
    import ctypes
    lib = attn.load_library()
    q8 = torch.zeros(1, 1, 128, 128, dtype=torch.float8_e4m3fn, device="cuda")
    o = torch.empty(1, 1, 128, 128, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(1, 1, 128, dtype=torch.float32, device="cuda")
    ws = torch.empty(attn.fp8_workspace_bytes(1, 1, 128, 128), dtype=torch.uint8, device="cuda")
    p = q8.data_ptr()
    args = lambda d, dsc, wsb: (p, p, p, dsc, 1.0, 1.0, o.data_ptr(), lse.data_ptr(), 1, 1, 128, d,
                                0, 0.1, ws.data_ptr(), wsb, None)
    assert lib.attn_fwd_fp8(*args(96, 1.0, ws.numel())) == ATTN_ERR_HEADDIM
    assert lib.attn_fwd_fp8(*args(128, 0.0, ws.numel())) == ATTN_ERR_SCALE
    assert lib.attn_fwd_fp8(*args(128, float("nan"), ws.numel())) == ATTN_ERR_SCALE
    assert lib.attn_fwd_fp8(*args(128, 1.0, ws.numel() - 1)) == ATTN_ERR_WORKSPACE
    assert lib.attn_fwd_fp8(*args(128, 1.0, ws.numel())) == 0
    torch.cuda.synchronize()
    assert attn.device_status(reset=True) == 0
