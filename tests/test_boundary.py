"""Host-side tests of the C ABI: the library loads, exports every function the
header declares, and rejects bad arguments before touching CUDA (so these run
on a machine without a GPU)."""
import ctypes
import math

import pytest
import torch

import exact_attention_127_b200 as attn
from exact_attention_127_b200 import _lib

OK, NULL, ALIGN, HEADDIM, SHAPE, SCALE = 0, -1, -2, -3, -4, -5
OVERLAP, WORKSPACE = -10, -11


@pytest.fixture(scope="module")
def lib():
    return attn.load_library()


def test_exports_every_header_function(lib):
    names = attn.header_functions()
    assert {"attn_fwd", "attn_fwd_host", "attn_fwd_host_workspace_bytes", "attn_device_status",
            "attn_status_str", "attn_version"} <= set(names)
    for name in names:
        assert hasattr(lib, name), f"{name} declared in the header but not exported"


def test_status_strings(lib):
    for code in range(0, -12, -1):
        s = attn.status_str(code)
        assert s and s != "unknown status"
    assert attn.status_str(-99) == "unknown status"
    assert attn.version()


FAKE = 0x10000   # 16-byte aligned, never dereferenced: validation fails first


def _call(lib, q=FAKE, k=FAKE + 0x100000, v=FAKE + 0x200000, o=FAKE + 0x300000,
          lse=FAKE + 0x400000, B=1, H=1, N=128, d=64, causal=0, scale=0.125):
    return lib.attn_fwd(q, k, v, o, lse, B, H, N, d, causal, scale, None)


def test_rejects_bad_head_dim(lib):
    for d in (0, 32, 96, 256):
        assert _call(lib, d=d) == HEADDIM


def test_rejects_bad_shapes(lib):
    assert _call(lib, B=-1) == SHAPE
    assert _call(lib, N=-5) == SHAPE
    assert _call(lib, N=2**31) == SHAPE
    assert _call(lib, B=2**20, H=2**20) == SHAPE


def test_rejects_bad_scale(lib):
    for s in (0.0, -1.0, math.inf, math.nan):
        assert _call(lib, scale=s) == SCALE


def test_rejects_null_and_misaligned(lib):
    assert _call(lib, q=None) == NULL
    assert _call(lib, lse=None) == NULL
    assert _call(lib, k=FAKE + 8) == ALIGN
    assert _call(lib, o=FAKE + 0x300002) == ALIGN


def test_rejects_overlapping_outputs(lib):
    assert _call(lib, o=FAKE) == OVERLAP                   # o on top of q
    assert _call(lib, lse=FAKE + 0x300000 + 64) == OVERLAP  # lse inside o


def test_other_entry_points_reject_overlaps(lib):
    """attn_bwd, attn_standard and attn_decode check overlaps before any launch."""
    big = 1 << 40
    ws = FAKE + 0x10000000                      # 256-byte aligned, far from the tensors
    a = [FAKE + 0x100000 * i for i in range(9)]  # q k v o dout lse dq dk dv
    assert lib.attn_bwd(*a, 1, 1, 128, 64, 0, 0.1, ws, big, None) != OVERLAP
    b = list(a)
    b[6] = a[0]                                  # dq on top of q
    assert lib.attn_bwd(*b, 1, 1, 128, 64, 0, 0.1, ws, big, None) == OVERLAP
    b = list(a)
    b[8] = a[7] + 64                             # dv inside dk
    assert lib.attn_bwd(*b, 1, 1, 128, 64, 0, 0.1, ws, big, None) == OVERLAP
    assert lib.attn_bwd(*a, 1, 1, 128, 64, 0, 0.1, a[3], big, None) == OVERLAP   # workspace on o
    assert lib.attn_standard(a[0], a[1], a[2], a[1], a[4], 1, 1, 128, 64, 0, 0.1, ws, big, None) == OVERLAP
    assert lib.attn_decode(a[0], a[1], a[2], a[2] + 32, a[4], 1, 1, 128, 64, 0.1, ws, big, None) == OVERLAP
    assert lib.attn_decode(a[0], a[1], a[2], a[3], a[4], 1, 1, 128, 64, 0.1, a[1], big, None) == OVERLAP


def test_empty_problem_is_ok_without_pointers(lib):
    assert _call(lib, q=None, k=None, v=None, o=None, lse=None, B=0) == OK
    assert _call(lib, q=None, k=None, v=None, o=None, lse=None, N=0) == OK


@pytest.mark.parametrize("B,N", [(0, 100), (1, 0)])
def test_every_entry_point_accepts_an_empty_problem(lib, B, N):
    """B * H * N = 0 is a valid problem with nothing to compute: every entry
    point returns ATTN_OK before it looks at a pointer or the device."""
    n = None
    assert lib.attn_fwd_host(n, n, n, n, n, B, 2, N, 64, 1, 0.125, n, 0, n) == OK
    assert lib.attn_fwd_fp8(n, n, n, 1.0, 1.0, 1.0, n, n, B, 2, N, 128, 1, 0.125, n, 0, n) == OK
    assert lib.attn_bwd(n, n, n, n, n, n, n, n, n, B, 2, N, 64, 1, 0.125, n, 0, n) == OK
    assert lib.attn_standard(n, n, n, n, n, B, 2, N, 64, 0, 0.125, n, 0, n) == OK
    # decode follows the same rule; over N = 0 cached keys it writes nothing
    assert lib.attn_decode(n, n, n, n, n, B, 2, N, 64, 0.125, n, 0, n) == OK


def test_host_entry_point_validation(lib):
    f = lib.attn_fwd_host
    assert lib.attn_fwd_host_workspace_bytes(1, 1, 128, 96) == 0
    need = lib.attn_fwd_host_workspace_bytes(1, 2, 100, 64)
    assert need >= 4 * 2 * 100 * 64 * 2 + 4 * 200
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 2, 100, 64, 0, 0.125, None, need, None) == WORKSPACE
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 2, 100, 64, 0, 0.125, 0x1000, need - 1, None) == WORKSPACE
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 2, 100, 64, 0, 0.125, 0x1010, need, None) == WORKSPACE
    assert f(None, FAKE, FAKE, FAKE, FAKE, 1, 2, 100, 64, 0, 0.125, 0x1000, need, None) == NULL
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 2, 100, 80, 0, 0.125, 0x1000, need, None) == HEADDIM


def test_python_binding_checks_metadata():
    q = torch.zeros(1, 1, 8, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        attn.attn_fwd(q.float(), q, q)
    with pytest.raises(ValueError):
        attn.attn_fwd(q, q, q)                       # CPU tensors on the device entry point
    with pytest.raises(ValueError):
        attn.attn_fwd_host(q, q, q[:, :, :4].contiguous())
    with pytest.raises(ValueError):
        attn.attn_fwd_host(q.transpose(2, 3), q, q)


def test_library_missing_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(_lib, "_lib", None)
    monkeypatch.setattr(_lib, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="no CPU fallback"):
        _lib.load_library()
