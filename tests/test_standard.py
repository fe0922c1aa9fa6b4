"""The unfused three-kernel standard path (S and P through device memory):
the same parity bar against the fp64 oracle as the fused kernel, plus the
fused kernel and the standard path agree with each other."""
import math

import numpy as np
import pytest
import torch

import exact_attention_127_b200 as attn
import oracle
from exact_attention_127_b200 import inputs

O_MAX_ABS, O_REL_L2, LSE_MAX_ABS = 2e-2, 5e-3, 1e-3
FAKE = 0x10000


def test_standard_validation_on_host():
    lib = attn.load_library()
    args = (FAKE, FAKE + 0x100000, FAKE + 0x200000, FAKE + 0x300000, FAKE + 0x400000)
    big = 1 << 40
    assert lib.attn_standard(*args, 1, 1, 40000, 64, 0, 0.1, FAKE + 0x500000, big, None) == -4
    assert lib.attn_standard(*args, 1, 70000, 16, 64, 0, 0.1, FAKE + 0x500000, big, None) == -4
    assert lib.attn_standard(*args, 1, 1, 100, 64, 0, 0.1, None, big, None) == -11
    assert lib.attn_standard(*args, 1, 1, 100, 64, 0, 0.1, FAKE + 0x500000, 1024, None) == -11
    assert lib.attn_standard_workspace_bytes(2, 3, 100, 64) == 2 * 3 * 128 * 128 * 4
    assert lib.attn_standard_workspace_bytes(1, 1, 40000, 64) == 0


@pytest.mark.gpu
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 100, 128, 300, 1000])
def test_standard_matches_oracle(N, d, causal):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    q, k, v = inputs.make_qkv(2, 2, N, d, seed=300 + N)
    o, lse = attn.attn_standard(q.cuda(), k.cuda(), v.cuda(), causal=causal)
    torch.cuda.synchronize()
    assert attn.device_status(reset=True) == 0
    O, L = oracle.attention_rows(q, k, v, causal, 1 / math.sqrt(d))
    of = o.cpu().reshape(4, N, d).double().numpy()
    lf = lse.cpu().reshape(4, N).double().numpy()
    assert np.abs(of - O).max() <= O_MAX_ABS
    assert np.linalg.norm(of - O) / np.linalg.norm(O) <= O_REL_L2
    assert np.abs(lf - L).max() <= LSE_MAX_ABS


@pytest.mark.gpu
def test_standard_and_fused_agree_on_a_workload():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    w = inputs.WORKLOADS["b8h16_n2048_d64"]
    q, k, v = (t.cuda() for t in inputs.workload_inputs(w))
    o1, l1 = attn.attn_fwd(q, k, v, causal=True)
    o2, l2 = attn.attn_standard(q, k, v, causal=True)
    torch.cuda.synchronize()
    assert attn.device_status(reset=True) == 0
    assert (o1.float() - o2.float()).abs().max().item() <= 2 * O_MAX_ABS
    assert (l1 - l2).abs().max().item() <= 2 * LSE_MAX_ABS


@pytest.mark.gpu
@pytest.mark.parametrize("N,causal", [(2049, True), (4096, False), (4097, True), (8192, True),
                                      (8193, False), (16384, True), (16385, True)])
def test_standard_long_rows_sampled(N, causal):
    """Rows longer than 2048 keys take the CTA-per-row softmax, instantiated for
    4, 8, 16 or 32 float4 per thread by row length: each class and its edges,
    checked on sampled rows (boundary rows plus seeded draws) of two heads."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    d = 64
    q, k, v = inputs.make_qkv(1, 2, N, d, seed=400 + N)
    o, lse = attn.attn_standard(q.cuda(), k.cuda(), v.cuda(), causal=causal)
    torch.cuda.synchronize()
    assert attn.device_status(reset=True) == 0
    rng = np.random.default_rng(N)
    rows = np.unique(np.concatenate([[0, 1, 127, 128, N // 2, N - 2, N - 1],
                                     rng.integers(0, N, 57)])).astype(np.int64)
    O, L = oracle.attention_rows(q, k, v, causal, 1 / math.sqrt(d), rows=rows)
    of = o.cpu().reshape(2, N, d)[:, torch.from_numpy(rows)].double().numpy()
    lf = lse.cpu().reshape(2, N)[:, torch.from_numpy(rows)].double().numpy()
    assert np.abs(of - O).max() <= O_MAX_ABS
    assert np.linalg.norm(of - O) / np.linalg.norm(O) <= O_REL_L2
    assert np.abs(lf - L).max() <= LSE_MAX_ABS
