"""Failure detection without a GPU fault: every wait in the kernel is bounded.

The test hooks attn_fwd_test_wait_timeout and attn_decode_test_wait_timeout run
the forward and decode kernels with their K/V loads withheld and a 20 ms limit
on each wait.  The waits run out, the kernel
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
