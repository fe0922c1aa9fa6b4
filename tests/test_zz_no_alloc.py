"""The allocation-free decode entry point, attn_decode_noalloc.

Some callers cannot allocate device memory themselves: a plugin whose host
application owns every device allocation through its own pool, or a loop that
must not call cudaMalloc (which can synchronise the device) once it runs.  For
them the library keeps the decode partial results in a fixed 8 MiB static
device buffer instead of a caller-provided workspace.

The GPU tests call that entry point through the C ABI:
- twice in a row, with different shapes, checking each result element by
  element against the fp64 oracle (attention_qk) and against the workspace
  entry point attn_decode, within the tolerances of the other parity tests;
- in a child process, in the primary context, a second context and the primary
  one again: the buffer has its own address in each context, so the library
  must look it up again after every switch (the same holds after a
  cudaDeviceReset, which this test does not do so as not to disturb the
  process's other users of the device).
This file's name makes pytest collect it last, so a run that stops at the
first failure has run every other test first; it also passes on its own in a
fresh process.
"""
import ctypes
import math
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import exact_attention_127_b200 as attn
import oracle
from exact_attention_127_b200 import inputs

O_MAX_ABS, O_REL_L2, LSE_MAX_ABS = 2e-2, 5e-3, 1e-3
ATTN_ERR_WORKSPACE = -11
HERE = os.path.dirname(os.path.abspath(__file__))


def _lib():
    lib = attn.load_library()
    vp, i64 = ctypes.c_void_p, ctypes.c_int64
    lib.attn_decode_noalloc.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i64,
                                        ctypes.c_float, vp]
    lib.attn_decode_noalloc.restype = ctypes.c_int
    lib.attn_decode_noalloc_scratch_bytes.argtypes = []
    lib.attn_decode_noalloc_scratch_bytes.restype = ctypes.c_size_t
    return lib


def test_no_alloc_limit_is_enforced_on_host():
    lib = _lib()
    assert lib.attn_decode_noalloc_scratch_bytes() == 8 << 20
    # a shape whose partials exceed the static buffer is refused before any launch
    B, H, N, d = 256, 128, 4096, 128
    assert attn.decode_workspace_bytes(B, H, N, d) > 8 << 20
    fake = 0x10000
    rc = lib.attn_decode_noalloc(fake, fake + 0x100000, fake + 0x200000, fake + 0x300000,
                                 fake + 0x400000, B, H, N, d, 0.1, None)
    assert rc == ATTN_ERR_WORKSPACE


def _close(a, b, what):
    err = np.abs(a - b).max()
    rel = np.linalg.norm(a - b) / np.linalg.norm(b)
    assert err <= O_MAX_ABS and rel <= O_REL_L2, f"{what}: max|dO|={err:.3e} relL2={rel:.3e}"


@pytest.mark.gpu
def test_no_alloc_decode_matches_oracle_twice():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    lib = _lib()
    stream = torch.cuda.current_stream()
    for (B, H, N, d, seed) in [(2, 3, 3000, 128, 41), (1, 2, 515, 64, 42)]:
        assert attn.decode_workspace_bytes(B, H, N, d) <= lib.attn_decode_noalloc_scratch_bytes()
        q, k, v = inputs.make_decode_qkv(B, H, N, d, seed)
        qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
        o = torch.empty_like(qd)
        lse = torch.empty((B, H), dtype=torch.float32, device="cuda")
        rc = lib.attn_decode_noalloc(qd.data_ptr(), kd.data_ptr(), vd.data_ptr(), o.data_ptr(),
                                     lse.data_ptr(), B, H, N, d, 1.0 / math.sqrt(d),
                                     stream.cuda_stream)
        assert rc == 0
        torch.cuda.synchronize()
        assert attn.device_status(reset=True) == 0
        a = o.double().cpu().numpy().reshape(B * H, 1, d)
        la = lse.double().cpu().numpy().reshape(B * H, 1)
        O, L = oracle.attention_qk(q, k, v, 1.0 / math.sqrt(d))
        _close(a, O, "against the oracle")
        assert np.abs(la - L).max() <= LSE_MAX_ABS
        o_ws, l_ws = attn.attn_decode(qd, kd, vd)       # the workspace entry point
        _close(a, o_ws.double().cpu().numpy().reshape(B * H, 1, d), "against attn_decode")
        assert (lse.double() - l_ws.double()).abs().max().item() <= LSE_MAX_ABS


@pytest.mark.gpu
def test_no_alloc_decode_after_context_switches():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    res = subprocess.run([sys.executable, os.path.join(HERE, "no_alloc_contexts.py")],
                         capture_output=True, text=True, timeout=300)
    assert res.returncode == 0 and res.stdout.strip().endswith("ok"), res.stdout + res.stderr
