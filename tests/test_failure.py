"""Failure detection without a GPU fault: every wait in the kernel is bounded.

The test hooks attn_fwd_test_wait_timeout, attn_decode_test_wait_timeout and
attn_bwd_test_wait_timeout run the forward, decode and backward kernels with
their loads withheld and a 20 ms limit on each wait.  The waits run out, the kernel
records ATTN_ERR_TIMEOUT in the device status word, frees its tensor memory
and exits; the context stays usable for the next call.
"""
import math
import time

import numpy as np
import pytest
import torch

import exact_attention_127_b200 as attn
import oracle
from exact_attention_127_b200 import inputs

ATTN_ERR_TIMEOUT = -8
ATTN_ERR_HEADDIM = -3


def test_hook_validates_arguments_on_host():
    lib = attn.load_library()
    fake = 0x10000
    rc = lib.attn_fwd_test_wait_timeout(fake, fake + 0x100000, fake + 0x200000, fake + 0x300000,
                                        fake + 0x400000, 1, 1, 128, 96, None)
    assert rc == ATTN_ERR_HEADDIM
    rc = lib.attn_decode_test_wait_timeout(fake, fake + 0x100000, fake + 0x200000, fake + 0x300000,
                                           fake + 0x400000, 1, 1, 128, 96, fake + 0x500000, 1 << 20,
                                           None)
    assert rc == ATTN_ERR_HEADDIM
    a = [fake + 0x100000 * i for i in range(9)]
    rc = lib.attn_bwd_test_wait_timeout(*a, 1, 1, 128, 96, 0, fake + 0x1000000, 1 << 30, None)
    assert rc == ATTN_ERR_HEADDIM


@pytest.mark.gpu
def test_bounded_wait_runs_out_and_context_survives():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    lib = attn.load_library()
    assert attn.device_status(reset=True) == 0
    q, k, v = (t.cuda() for t in inputs.make_qkv(1, 2, 300, 64, seed=31))
    o = torch.empty_like(q)
    lse = torch.empty(1, 2, 300, dtype=torch.float32, device="cuda")
    t0 = time.perf_counter()
    rc = lib.attn_fwd_test_wait_timeout(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                        lse.data_ptr(), 1, 2, 300, 64,
                                        torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    status = attn.device_status(reset=True)
    elapsed = time.perf_counter() - t0
    assert status == ATTN_ERR_TIMEOUT
    assert elapsed < 10.0
    assert attn.device_status(reset=True) == 0      # the word was cleared
    # the next ordinary call runs normally and is correct
    qc, kc, vc = inputs.make_qkv(1, 2, 300, 64, seed=32)
    o2, l2 = attn.attn_fwd(qc.cuda(), kc.cuda(), vc.cuda(), causal=True)
    torch.cuda.synchronize()
    assert attn.device_status(reset=True) == 0
    O, L = oracle.attention_rows(qc, kc, vc, True, 1 / math.sqrt(64))
    assert np.abs(o2.cpu().reshape(2, 300, 64).double().numpy() - O).max() <= 2e-2
    assert np.abs(l2.cpu().reshape(2, 300).double().numpy() - L).max() <= 1e-3


@pytest.mark.gpu
def test_decode_bounded_wait_runs_out_and_context_survives():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    lib = attn.load_library()
    assert attn.device_status(reset=True) == 0
    B, H, N, d = 2, 3, 3000, 128
    q, k, v = (t.cuda() for t in inputs.make_decode_qkv(B, H, N, d, 33))
    o = torch.empty_like(q)
    lse = torch.empty(B, H, dtype=torch.float32, device="cuda")
    ws = torch.empty(attn.decode_workspace_bytes(B, H, N, d), dtype=torch.uint8, device="cuda")
    t0 = time.perf_counter()
    rc = lib.attn_decode_test_wait_timeout(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                           lse.data_ptr(), B, H, N, d, ws.data_ptr(), ws.numel(),
                                           torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    status = attn.device_status(reset=True)
    elapsed = time.perf_counter() - t0
    assert status == ATTN_ERR_TIMEOUT
    assert elapsed < 10.0
    assert attn.device_status(reset=True) == 0
    # the next ordinary decode call runs normally and is correct
    o2, l2 = attn.attn_decode(q, k, v)
    torch.cuda.synchronize()
    assert attn.device_status(reset=True) == 0
    O, L = oracle.attention_qk(q.cpu(), k.cpu(), v.cpu(), 1.0 / math.sqrt(d))
    assert np.abs(o2.cpu().reshape(B * H, 1, d).double().numpy() - O).max() <= 2e-2
    assert np.abs(l2.cpu().reshape(B * H, 1).double().numpy() - L).max() <= 1e-3


@pytest.mark.gpu
@pytest.mark.parametrize("d,causal", [(64, False), (128, True)])
def test_backward_bounded_wait_runs_out_and_context_survives(d, causal):
    """The backward kernel with its loads withheld: every role's wait runs out
    (the MMA warp's on K/V, the P/dS warps' on S^T, the readout's on the dQ
    partial), ATTN_ERR_TIMEOUT is recorded, and the next call is correct."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    lib = attn.load_library()
    assert attn.device_status(reset=True) == 0
    B, H, N = 1, 2, 300
    q, k, v = (t.cuda() for t in inputs.make_qkv(B, H, N, d, seed=34))
    dout = inputs.make_qkv(B, H, N, d, seed=35)[0].cuda()
    o, lse = attn.attn_fwd(q, k, v, causal=causal, scale=0.125)
    dq, dk, dv = (torch.empty_like(q) for _ in range(3))
    ws = torch.empty(attn.bwd_workspace_bytes(B, H, N, d), dtype=torch.uint8, device="cuda")
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    rc = lib.attn_bwd_test_wait_timeout(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                        dout.data_ptr(), lse.data_ptr(), dq.data_ptr(), dk.data_ptr(),
                                        dv.data_ptr(), B, H, N, d, int(causal), ws.data_ptr(),
                                        ws.numel(), torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    status = attn.device_status(reset=True)
    elapsed = time.perf_counter() - t0
    assert status == ATTN_ERR_TIMEOUT
    assert elapsed < 10.0
    assert attn.device_status(reset=True) == 0
    # the next ordinary backward call runs normally and matches the oracle
    dq2, dk2, dv2 = attn.attn_bwd(q, k, v, o, lse, dout, causal=causal, scale=0.125, workspace=ws)
    torch.cuda.synchronize()
    assert attn.device_status(reset=True) == 0
    ref = oracle.attention_backward(q.cpu(), k.cpu(), v.cpu(), dout.cpu(), causal, 0.125)
    for g, r in zip((dq2, dk2, dv2), ref):
        gf = g.cpu().reshape(B * H, N, d).double().numpy()
        assert np.linalg.norm(gf - r) <= 1e-2 * np.linalg.norm(r)

