"""ctypes binding of libattn127.so: argument marshalling only.

Every step of the attention computation runs in the library's CUDA kernel;
this module only checks tensor metadata, allocates outputs through PyTorch and
forwards pointers.  There is no fallback: if the library is missing, or the
device is not an sm_100 GPU, calls raise.
"""
from __future__ import annotations

import ctypes
import math
import os
import re

import torch

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libattn127.so")
HEADER_PATH = os.path.join(os.path.dirname(PKG), "include", "attn_fwd.h")

ATTN_OK = 0


class AttnError(RuntimeError):
    """A non-zero status returned by the C library."""

    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_str(status)} (status {status})")


_lib = None


def load_library():
    """Load (once) and return the ctypes handle of libattn127.so."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            f"CUDA library {LIB_PATH} is missing; build it with "
            "`python -m exact_attention_127_b200.build` (there is no CPU fallback)")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i64, c_int = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    lib.attn_fwd.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i64, c_int, ctypes.c_float, vp]
    lib.attn_fwd.restype = c_int
    lib.attn_fwd_host.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i64, c_int, ctypes.c_float,
                                  vp, ctypes.c_size_t, vp]
    lib.attn_fwd_host.restype = c_int
    lib.attn_fwd_host_workspace_bytes.argtypes = [i64, i64, i64, i64]
    lib.attn_fwd_host_workspace_bytes.restype = ctypes.c_size_t
    lib.attn_device_status.argtypes = [vp, c_int]
    lib.attn_device_status.restype = c_int
    lib.attn_bwd_workspace_bytes.argtypes = [i64, i64, i64, i64]
    lib.attn_bwd_workspace_bytes.restype = ctypes.c_size_t
    lib.attn_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i64, i64, i64, i64, c_int,
                             ctypes.c_float, vp, ctypes.c_size_t, vp]
    lib.attn_bwd.restype = c_int
    lib.attn_standard_workspace_bytes.argtypes = [i64, i64, i64, i64]
    lib.attn_standard_workspace_bytes.restype = ctypes.c_size_t
    lib.attn_standard.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i64, c_int, ctypes.c_float,
                                  vp, ctypes.c_size_t, vp]
    lib.attn_standard.restype = c_int
    lib.attn_fwd_fp8_workspace_bytes.argtypes = [i64, i64, i64, i64]
    lib.attn_fwd_fp8_workspace_bytes.restype = ctypes.c_size_t
    f32 = ctypes.c_float
    lib.attn_fwd_fp8.argtypes = [vp, vp, vp, f32, f32, f32, vp, vp, i64, i64, i64, i64, c_int, f32,
                                 vp, ctypes.c_size_t, vp]
    lib.attn_fwd_fp8.restype = c_int
    lib.attn_decode_workspace_bytes.argtypes = [i64, i64, i64, i64]
    lib.attn_decode_workspace_bytes.restype = ctypes.c_size_t
    lib.attn_decode.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i64, ctypes.c_float, vp,
                                ctypes.c_size_t, vp]
    lib.attn_decode.restype = c_int
    lib.attn_fwd_test_wait_timeout.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i64, vp]
    lib.attn_fwd_test_wait_timeout.restype = c_int
    lib.attn_decode_test_wait_timeout.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i64, vp,
                                                  ctypes.c_size_t, vp]
    lib.attn_decode_test_wait_timeout.restype = c_int
    lib.attn_bwd_test_wait_timeout.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i64, i64, i64, i64,
                                               c_int, vp, ctypes.c_size_t, vp]
    lib.attn_bwd_test_wait_timeout.restype = c_int
    i32p = ctypes.POINTER(ctypes.c_int32)
    lib.attn_fwd_schedule.argtypes = [i64, i64, i64, c_int, c_int, i32p, i32p, i64]
    lib.attn_fwd_schedule.restype = i64
    lib.attn_status_str.argtypes = [c_int]
    lib.attn_status_str.restype = ctypes.c_char_p
    lib.attn_version.argtypes = []
    lib.attn_version.restype = ctypes.c_char_p
    _lib = lib
    return lib


def header_functions(path: str = HEADER_PATH):
    """Names of the functions the public header declares."""
    text = open(path).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(attn_\w+)\s*\(", text)))


def status_str(status: int) -> str:
    return load_library().attn_status_str(int(status)).decode()


def version() -> str:
    return load_library().attn_version().decode()


def _stream_handle(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream)


def _check_inputs(q, k, v, device_expected: bool):
    for name, t in (("q", q), ("k", k), ("v", v)):
        if not isinstance(t, torch.Tensor):
            raise TypeError(f"{name} must be a torch.Tensor")
        if t.dtype != torch.bfloat16:
            raise ValueError(f"{name} must be bfloat16, got {t.dtype}")
        if t.dim() != 4:
            raise ValueError(f"{name} must be [B, H, N, d], got shape {tuple(t.shape)}")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
        if device_expected and not t.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor")
        if not device_expected and t.is_cuda:
            raise ValueError(f"{name} must be a CPU tensor")
    if not (q.shape == k.shape == v.shape):
        raise ValueError("q, k, v must share one [B, H, N, d] shape")
    if device_expected and not (q.device == k.device == v.device):
        raise ValueError("q, k, v must be on one device")


def attn_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, causal: bool = False,
             scale: float | None = None, out: torch.Tensor | None = None,
             lse: torch.Tensor | None = None, stream=None):
    """O = softmax(scale*QK^T [+causal mask]) V and LSE, on the GPU.

    q, k, v: bf16 CUDA tensors [B, H, N, d], contiguous, d in {64, 128}.
    Returns (o bf16 [B, H, N, d], lse fp32 [B, H, N]).  Asynchronous on
    `stream` (default: torch's current stream).
    """
    _check_inputs(q, k, v, device_expected=True)
    B, H, N, d = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    if out.shape != q.shape or out.dtype != torch.bfloat16 or not out.is_contiguous():
        raise ValueError("out must be a contiguous bf16 tensor shaped like q")
    if tuple(lse.shape) != (B, H, N) or lse.dtype != torch.float32 or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous fp32 [B, H, N] tensor")
    lib = load_library()
    with torch.cuda.device(q.device):
        rc = lib.attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                          lse.data_ptr(), B, H, N, d, int(bool(causal)), float(scale),
                          _stream_handle(stream))
    if rc != ATTN_OK:
        raise AttnError(rc, "attn_fwd")
    return out, lse


def fwd_schedule(B: int, H: int, N: int, causal: bool, grid: int):
    """The forward kernel's static schedule (host only, no GPU needed).

    Returns (cta, slot): int32 tensors of B*H*ceil(N/256) entries; unit
    u = bh*ceil(N/256) + pair runs on CTA cta[u] as its slot[u]-th unit.
    """
    n_units = B * H * ((N + 255) // 256)
    cta = torch.full((max(n_units, 1),), -1, dtype=torch.int32)
    slot = torch.full((max(n_units, 1),), -1, dtype=torch.int32)
    i32p = ctypes.POINTER(ctypes.c_int32)
    rc = load_library().attn_fwd_schedule(B, H, N, int(bool(causal)), int(grid),
                                          ctypes.cast(cta.data_ptr(), i32p),
                                          ctypes.cast(slot.data_ptr(), i32p), cta.numel())
    if rc < 0:
        raise AttnError(int(rc), "attn_fwd_schedule")
    if rc != n_units:
        raise RuntimeError(f"attn_fwd_schedule visited {rc} units, expected {n_units}")
    return cta[:n_units], slot[:n_units]


def host_workspace_bytes(B: int, H: int, N: int, d: int) -> int:
    return int(load_library().attn_fwd_host_workspace_bytes(B, H, N, d))


def attn_fwd_host(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, causal: bool = False,
                  scale: float | None = None, out: torch.Tensor | None = None,
                  lse: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
                  device=None, stream=None, synchronize: bool = True):
    """The same operation on CPU tensors (pinned for asynchronous copies).

    The library copies q, k, v to `workspace` on the device, runs the kernel
    and copies o and lse back, all on one stream.  Returns (o, lse) as CPU
    tensors; with synchronize=False the caller must synchronise the stream.
    """
    _check_inputs(q, k, v, device_expected=False)
    B, H, N, d = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    device = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    pin = q.is_pinned()
    if out is None:
        out = torch.empty(q.shape, dtype=torch.bfloat16, pin_memory=pin)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, pin_memory=pin)
    need = host_workspace_bytes(B, H, N, d)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=device)
    lib = load_library()
    with torch.cuda.device(device):
        handle = _stream_handle(stream)
        rc = lib.attn_fwd_host(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                               lse.data_ptr(), B, H, N, d, int(bool(causal)), float(scale),
                               workspace.data_ptr(), workspace.numel(), handle)
        if rc != ATTN_OK:
            raise AttnError(rc, "attn_fwd_host")
        if synchronize:
            if stream is None:
                torch.cuda.current_stream(device).synchronize()
            elif hasattr(stream, "synchronize"):
                stream.synchronize()
            else:
                torch.cuda.synchronize(device)
    return out, lse


def bwd_workspace_bytes(B: int, H: int, N: int, d: int) -> int:
    return int(load_library().attn_bwd_workspace_bytes(B, H, N, d))


def attn_bwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o: torch.Tensor,
             lse: torch.Tensor, dout: torch.Tensor, causal: bool = False,
             scale: float | None = None, workspace: torch.Tensor | None = None, stream=None):
    """Gradients (dq, dk, dv) of the forward pass for upstream gradient dout,
    recomputed from the saved lse (o, lse from attn_fwd with the same inputs)."""
    _check_inputs(q, k, v, device_expected=True)
    for name, t in (("o", o), ("dout", dout)):
        if t.shape != q.shape or t.dtype != torch.bfloat16 or not t.is_contiguous() or not t.is_cuda:
            raise ValueError(f"{name} must be a contiguous bf16 CUDA tensor shaped like q")
    B, H, N, d = q.shape
    if tuple(lse.shape) != (B, H, N) or lse.dtype != torch.float32 or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous fp32 [B, H, N] tensor")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dq, dk, dv = (torch.empty_like(q) for _ in range(3))
    if workspace is None:
        workspace = torch.empty(max(bwd_workspace_bytes(B, H, N, d), 1), dtype=torch.uint8,
                                device=q.device)
    lib = load_library()
    with torch.cuda.device(q.device):
        rc = lib.attn_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), dout.data_ptr(),
                          lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, H, N, d,
                          int(bool(causal)), float(scale), workspace.data_ptr(), workspace.numel(),
                          _stream_handle(stream))
    if rc != ATTN_OK:
        raise AttnError(rc, "attn_bwd")
    return dq, dk, dv


def standard_workspace_bytes(B: int, H: int, N: int, d: int) -> int:
    return int(load_library().attn_standard_workspace_bytes(B, H, N, d))


def attn_standard(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, causal: bool = False,
                  scale: float | None = None, out: torch.Tensor | None = None,
                  lse: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
                  stream=None):
    """The unfused three-kernel path (S and P through device memory), for
    comparison with attn_fwd.  Same inputs and outputs as attn_fwd."""
    _check_inputs(q, k, v, device_expected=True)
    B, H, N, d = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = torch.empty(max(standard_workspace_bytes(B, H, N, d), 1), dtype=torch.uint8,
                                device=q.device)
    lib = load_library()
    with torch.cuda.device(q.device):
        rc = lib.attn_standard(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                               lse.data_ptr(), B, H, N, d, int(bool(causal)), float(scale),
                               workspace.data_ptr(), workspace.numel(), _stream_handle(stream))
    if rc != ATTN_OK:
        raise AttnError(rc, "attn_standard")
    return out, lse


def fp8_workspace_bytes(B: int, H: int, N: int, d: int) -> int:
    return int(load_library().attn_fwd_fp8_workspace_bytes(B, H, N, d))


def attn_fwd_fp8(q8: torch.Tensor, k8: torch.Tensor, v8: torch.Tensor, q_descale: float = 1.0,
                 k_descale: float = 1.0, v_descale: float = 1.0, causal: bool = False,
                 scale: float | None = None, out: torch.Tensor | None = None,
                 lse: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
                 stream=None):
    """The forward pass on e4m3 inputs (torch.float8_e4m3fn [B, H, N, d] CUDA
    tensors, d in {64, 128}): the scores use q8*q_descale and k8*k_descale, the
    values v8*v_descale.  O (bf16) and LSE (fp32) as attn_fwd."""
    for name, t in (("q8", q8), ("k8", k8), ("v8", v8)):
        if not isinstance(t, torch.Tensor):
            raise TypeError(f"{name} must be a torch.Tensor")
        if t.dtype != torch.float8_e4m3fn:
            raise ValueError(f"{name} must be float8_e4m3fn, got {t.dtype}")
        if t.dim() != 4 or not t.is_contiguous() or not t.is_cuda:
            raise ValueError(f"{name} must be a contiguous CUDA [B, H, N, d] tensor")
    if not (q8.shape == k8.shape == v8.shape) or not (q8.device == k8.device == v8.device):
        raise ValueError("q8, k8, v8 must share one shape and device")
    B, H, N, d = q8.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty((B, H, N, d), dtype=torch.bfloat16, device=q8.device)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q8.device)
    if workspace is None:
        workspace = torch.empty(max(fp8_workspace_bytes(B, H, N, d), 1), dtype=torch.uint8,
                                device=q8.device)
    lib = load_library()
    with torch.cuda.device(q8.device):
        rc = lib.attn_fwd_fp8(q8.data_ptr(), k8.data_ptr(), v8.data_ptr(), float(q_descale),
                              float(k_descale), float(v_descale), out.data_ptr(), lse.data_ptr(),
                              B, H, N, d, int(bool(causal)), float(scale), workspace.data_ptr(),
                              workspace.numel(), _stream_handle(stream))
    if rc != ATTN_OK:
        raise AttnError(rc, "attn_fwd_fp8")
    return out, lse


def decode_workspace_bytes(B: int, H: int, N: int, d: int) -> int:
    return int(load_library().attn_decode_workspace_bytes(B, H, N, d))


def attn_decode(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, scale: float | None = None,
                out: torch.Tensor | None = None, lse: torch.Tensor | None = None,
                workspace: torch.Tensor | None = None, stream=None):
    """One query row per head against N cached keys (split-K/V decode).

    q: bf16 CUDA [B, H, 1, d] (or [B, H, d]); k, v: bf16 CUDA [B, H, N, d].
    Returns (o bf16 [B, H, 1, d] shaped like q, lse fp32 [B, H]).
    """
    for name, t in (("q", q), ("k", k), ("v", v)):
        if not isinstance(t, torch.Tensor) or t.dtype != torch.bfloat16 or not t.is_cuda:
            raise ValueError(f"{name} must be a bf16 CUDA tensor")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    if k.dim() != 4 or k.shape != v.shape:
        raise ValueError("k and v must share one [B, H, N, d] shape")
    B, H, N, d = k.shape
    if tuple(q.shape) not in ((B, H, 1, d), (B, H, d)):
        raise ValueError("q must be [B, H, 1, d] or [B, H, d]")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = torch.empty(max(decode_workspace_bytes(B, H, N, d), 1), dtype=torch.uint8,
                                device=q.device)
    lib = load_library()
    with torch.cuda.device(q.device):
        rc = lib.attn_decode(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                             lse.data_ptr(), B, H, N, d, float(scale), workspace.data_ptr(),
                             workspace.numel(), _stream_handle(stream))
    if rc != ATTN_OK:
        raise AttnError(rc, "attn_decode")
    return out, lse


def device_status(reset: bool = True, stream=None) -> int:
    """Synchronise `stream` and return (and by default clear) the device
    status word: 0, or the first in-kernel error code recorded."""
    return int(load_library().attn_device_status(_stream_handle(stream), int(bool(reset))))
