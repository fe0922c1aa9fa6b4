"""GPU parity: the CUDA kernel (through the C ABI) against the fp64 CPU oracle,
element by element, on the same seeded bf16 inputs.

Tolerances (fixed for the fused forward in bf16 with fp32 statistics):
max |dO| <= 2e-2, relative L2 error of O <= 5e-3, max |dLSE| <= 1e-3.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from exact_attention_127_b200 import inputs

pytestmark = pytest.mark.gpu

O_MAX_ABS = 2e-2
O_REL_L2 = 5e-3
LSE_MAX_ABS = 1e-3


@pytest.fixture(scope="module")
def attn():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import exact_attention_127_b200 as m
    m.load_library()
    assert m.device_status(reset=True) == 0
    return m


def _run(attn, q, k, v, causal, scale=None):
    qd, kd, vd = (t.cuda() for t in (q, k, v))
    o, lse = attn.attn_fwd(qd, kd, vd, causal=causal, scale=scale)
    torch.cuda.synchronize()
    assert attn.device_status(reset=True) == 0
    return o.cpu(), lse.cpu()


def _compare(o, lse, O_ref, L_ref, heads, rows, label=""):
    B, H, N, d = o.shape
    of = o.reshape(B * H, N, d)[heads][:, rows].double().numpy()
    lf = lse.reshape(B * H, N)[heads][:, rows].double().numpy()
    assert np.all(np.isfinite(of)) and np.all(np.isfinite(lf)), label
    err = np.abs(of - O_ref)
    rel = np.linalg.norm(of - O_ref) / max(np.linalg.norm(O_ref), 1e-30)
    lerr = np.abs(lf - L_ref)
    msg = f"{label}: max|dO|={err.max():.3e} relL2={rel:.3e} max|dLSE|={lerr.max():.3e}"
    assert err.max() <= O_MAX_ABS, msg
    assert rel <= O_REL_L2, msg
    assert lerr.max() <= LSE_MAX_ABS, msg
    return err.max(), rel, lerr.max()


def _full_check(attn, q, k, v, causal, scale=None, label=""):
    B, H, N, d = q.shape
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    o, lse = _run(attn, q, k, v, causal, scale)
    O_ref, L_ref = oracle.attention_rows(q, k, v, causal, scale)
    return _compare(o, lse, O_ref, L_ref, list(range(B * H)), np.arange(N), label)


# ---------------------------------------------------------------------------
# Edge shapes: empty/ragged tails, single tile, tile boundaries, two tiles
# per work unit with the second one partly or wholly past N.
# ---------------------------------------------------------------------------
EDGE_N = [1, 2, 127, 128, 129, 255, 256, 257, 300, 383, 384, 385, 1000]


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", EDGE_N)
def test_edge_shapes(attn, N, d, causal):
    q, k, v = inputs.make_qkv(1, 2, N, d, seed=100 + N)
    _full_check(attn, q, k, v, causal, label=f"N={N} d={d} causal={causal}")


@pytest.mark.parametrize("d", [64, 128])
def test_many_heads_more_units_than_sms(attn, d):
    # 3*70 heads x 1 unit: every CTA runs several units (snake schedule)
    q, k, v = inputs.make_qkv(3, 70, 200, d, seed=7)
    _full_check(attn, q, k, v, causal=True, label=f"many heads d={d}")


@pytest.mark.parametrize("causal", [False, True])
def test_non_default_scale(attn, causal):
    q, k, v = inputs.make_qkv(2, 3, 333, 64, seed=8)
    _full_check(attn, q, k, v, causal, scale=0.3, label="scale=0.3")


# ---------------------------------------------------------------------------
# The five workloads.  Small ones: every row.  Large ones: a seeded sample of
# >= 256 query rows per head, including tile- and diagonal-boundary rows.
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("name", inputs.WORKLOAD_ORDER)
def test_workload(attn, name):
    w = inputs.WORKLOADS[name]
    q, k, v = inputs.workload_inputs(w)
    o, lse = _run(attn, q, k, v, w.causal, w.scale)
    heads = list(range(w.B * w.H))
    rows = np.arange(w.N) if w.N <= 2048 else inputs.sample_rows(w.N, 256, w.seed)
    if name == "b8h16_n2048_d64":
        rows = inputs.sample_rows(w.N, 512, w.seed)
    O_ref, L_ref = oracle.attention_rows(q, k, v, w.causal, w.scale, rows=rows, heads=heads)
    _compare(o, lse, O_ref, L_ref, heads, rows, label=name)


# ---------------------------------------------------------------------------
# Special inputs with exact or closed-form answers
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("d", [64, 128])
def test_causal_row0_is_v0_exactly(attn, d):
    """Row 0 attends to key 0 only: P = 1, l = 1, so O_0 is v_0 bit for bit."""
    q, k, v = inputs.make_qkv(2, 2, 700, d, seed=9)
    o, lse = _run(attn, q, k, v, causal=True)
    assert torch.equal(o[:, :, 0], v[:, :, 0])
    s0 = (q[:, :, 0].double() * k[:, :, 0].double()).sum(-1) / math.sqrt(d)
    assert torch.allclose(lse[:, :, 0].double(), s0, atol=1e-4, rtol=0)


@pytest.mark.parametrize("causal", [False, True])
def test_zero_queries_average_values(attn, causal):
    q, k, v = inputs.make_qkv(1, 2, 517, 128, seed=10)
    q.zero_()
    o, lse = _run(attn, q, k, v, causal)
    vf = v.double()
    n = torch.arange(1, 518, dtype=torch.float64)
    if causal:
        ref = vf.cumsum(2) / n[None, None, :, None]
        lref = torch.log(n)[None, None].expand(1, 2, 517)
    else:
        ref = vf.mean(2, keepdim=True).expand_as(vf)
        lref = torch.full((1, 2, 517), math.log(517), dtype=torch.float64)
    assert (o.double() - ref).abs().max() <= O_MAX_ABS
    assert (lse.double() - lref).abs().max() <= LSE_MAX_ABS


def test_duplicated_keys(attn):
    q, k, v = inputs.make_qkv(1, 1, 640, 64, seed=11)
    k[:, :, 1::2] = k[:, :, 0::2]
    _full_check(attn, q, k, v, causal=False, label="duplicated keys")


@pytest.mark.parametrize("causal", [False, True])
def test_large_logits(attn, causal):
    """Peaked softmax (std of logits ~16): exercises the lazy rescale path."""
    q, k, v = inputs.make_qkv(1, 4, 1500, 128, seed=12, qk_std=4.0, v_dist="uniform")
    _full_check(attn, q, k, v, causal, label="large logits")


@pytest.mark.parametrize("N", [1024, 1100])
def test_large_logits_d64(attn, N):
    """d = 64, non-causal, peaked softmax: the rescale path of the d = 64 kernel
    on an even number of 128-row Q tiles (N = 1024) and with a ragged tail
    (N = 1100)."""
    q, k, v = inputs.make_qkv(1, 3, N, 64, seed=14, qk_std=4.0, v_dist="uniform")
    _full_check(attn, q, k, v, False, label=f"large logits d64 N={N}")


def test_increasing_scores_force_rescales(attn):
    """Scores that grow along the keys move the reference max in every block."""
    N, d = 1024, 64
    q = torch.zeros(1, 1, N, d)
    q[..., 0] = 1.0
    k = torch.zeros(1, 1, N, d)
    k[..., 0] = torch.linspace(0, 60, N)
    v = torch.randn(1, 1, N, d, generator=torch.Generator().manual_seed(13))
    q, k, v = (t.to(torch.bfloat16) for t in (q, k, v))
    _full_check(attn, q, k, v, causal=False, scale=1.0, label="growing scores")
    _full_check(attn, q, k, v, causal=True, scale=1.0, label="growing scores causal")


# ---------------------------------------------------------------------------
# Determinism, host-buffer entry point, outputs untouched past the tensors
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("causal", [False, True])
def test_deterministic(attn, causal):
    q, k, v = (t.cuda() for t in inputs.make_qkv(2, 4, 1111, 128, seed=14))
    o1, l1 = attn.attn_fwd(q, k, v, causal=causal)
    o2, l2 = attn.attn_fwd(q, k, v, causal=causal)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_host_entry_point_matches_device(attn):
    q, k, v = inputs.make_qkv(2, 3, 777, 64, seed=15)
    o_d, l_d = _run(attn, q, k, v, causal=True)
    qp, kp, vp = (t.pin_memory() for t in (q, k, v))
    o_h, l_h = attn.attn_fwd_host(qp, kp, vp, causal=True)
    assert attn.device_status(reset=True) == 0
    assert torch.equal(o_h, o_d) and torch.equal(l_h, l_d)


@pytest.mark.parametrize("causal", [False, True])
def test_host_entry_point_pipelined_matches_device(attn, causal):
    """Above 32 MB of inputs the host entry point pipelines the copies and the
    kernel over chunks of heads (11 heads: chunks of 2, 2, 2, 2, 2, 1); every
    head's result is computed as in one call, so the outputs are identical."""
    q, k, v = inputs.make_qkv(1, 11, 4500, 128, seed=17)
    o_d, l_d = _run(attn, q, k, v, causal=causal)
    qp, kp, vp = (t.pin_memory() for t in (q, k, v))
    o_h, l_h = attn.attn_fwd_host(qp, kp, vp, causal=causal)
    assert attn.device_status(reset=True) == 0
    assert torch.equal(o_h, o_d) and torch.equal(l_h, l_d)
    # a second call through the same helper streams, on a user stream
    s = torch.cuda.Stream()
    o_h2, l_h2 = attn.attn_fwd_host(qp, kp, vp, causal=causal, stream=s)
    assert torch.equal(o_h2, o_d) and torch.equal(l_h2, l_d)


def test_no_writes_outside_outputs(attn):
    q, k, v = (t.cuda() for t in inputs.make_qkv(1, 3, 300, 128, seed=16))
    B, H, N, d = q.shape
    o_big = torch.full((B * H * N * d + 4096,), 7.0, dtype=torch.bfloat16, device="cuda")
    l_big = torch.full((B * H * N + 1024,), 7.0, dtype=torch.float32, device="cuda")
    o = o_big[:B * H * N * d].view(B, H, N, d)
    lse = l_big[:B * H * N].view(B, H, N)
    attn.attn_fwd(q, k, v, causal=True, out=o, lse=lse)
    torch.cuda.synchronize()
    assert torch.all(o_big[B * H * N * d:] == 7.0)
    assert torch.all(l_big[B * H * N:] == 7.0)


def test_empty_batch_is_a_no_op(attn):
    q = torch.empty(0, 2, 128, 64, dtype=torch.bfloat16, device="cuda")
    o, lse = attn.attn_fwd(q, q, q)
    assert o.shape == q.shape and lse.shape == (0, 2, 128)
