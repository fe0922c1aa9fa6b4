"""The forward and backward entry points inside a CUDA graph.

For launch-bound shapes (a single 128-row tile) the host work of a call
(argument checks, tensor-map encoding, the launch) costs more than the kernel;
a caller that captures the call once in a CUDA graph and replays it pays only
the graph launch.  A call does nothing that breaks stream capture: no
allocation, no synchronisation, no copy to or from the host, and the kernel
parameters (tensor maps, schedule) are plain values.  Per-context setup (the
shared-memory attribute of each kernel) happens on the first call, which these
tests make before capturing, as a caller would.

Each test captures one call, then replays the graph on new inputs written
into the captured buffers and compares the result bit for bit with an eager
call on the same inputs.
"""
import pytest
import torch

import exact_attention_127_b200 as attn
from exact_attention_127_b200 import inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    attn.load_library()
    assert attn.device_status(reset=True) == 0
    return attn


def _capture(fn):
    """Run fn once eagerly on a side stream, then capture it in a graph."""
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        fn()
    torch.cuda.current_stream().wait_stream(side)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    return g


@pytest.mark.parametrize("shape,causal", [((1, 1, 128, 64), False), ((2, 3, 700, 128), True),
                                          ((1, 2, 1000, 64), False), ((1, 2, 777, 64), True)])
def test_forward_graph_replay_matches_eager(lib, shape, causal):
    B, H, N, d = shape
    q, k, v = (t.cuda() for t in inputs.make_qkv(B, H, N, d, seed=21))
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device="cuda")
    g = _capture(lambda: attn.attn_fwd(q, k, v, causal=causal, out=o, lse=lse))
    for seed in (22, 23):
        nq, nk, nv = inputs.make_qkv(B, H, N, d, seed=seed)
        q.copy_(nq)
        k.copy_(nk)
        v.copy_(nv)
        g.replay()
        torch.cuda.synchronize()
        o_ref, l_ref = attn.attn_fwd(q, k, v, causal=causal)
        torch.cuda.synchronize()
        assert torch.equal(o, o_ref) and torch.equal(lse, l_ref)
    assert attn.device_status(reset=True) == 0


@pytest.mark.parametrize("d,causal", [(64, False), (128, True)])
def test_backward_graph_replay_matches_eager(lib, d, causal):
    B, H, N = 1, 2, 600
    q, k, v = (t.cuda() for t in inputs.make_qkv(B, H, N, d, seed=31))
    dout = inputs.make_qkv(B, H, N, d, seed=32)[0].cuda()
    o, lse = attn.attn_fwd(q, k, v, causal=causal)
    ws = torch.empty(attn.bwd_workspace_bytes(B, H, N, d), dtype=torch.uint8, device="cuda")
    grads = {}

    def bwd():
        grads["g"] = attn.attn_bwd(q, k, v, o, lse, dout, causal, None, workspace=ws)

    g = _capture(bwd)
    dq, dk, dv = grads["g"]          # the graph's output buffers
    for seed in (33, 34):
        dout.copy_(inputs.make_qkv(B, H, N, d, seed=seed)[0])
        g.replay()
        torch.cuda.synchronize()
        rq, rk, rv = attn.attn_bwd(q, k, v, o, lse, dout, causal, None, workspace=ws)
        torch.cuda.synchronize()
        # dK and dV are formed within one CTA; dQ sums the K/V blocks' partials with
        # fp32 reduce-adds in whatever order they reach L2, so it may differ in the
        # last bf16 bit
        assert torch.equal(dk, rk) and torch.equal(dv, rv)
        assert (dq.float() - rq.float()).abs().max() <= 1e-2 * rq.float().abs().max()
    assert attn.device_status(reset=True) == 0
