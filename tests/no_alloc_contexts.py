"""Child process of tests/test_zz_no_alloc.py (run as a script, not collected).

Calls attn_decode_noalloc in three CUDA contexts in turn, with no PyTorch CUDA
use in this process: the device's primary context, a second context created
with the driver API, then the primary one again.  A __device__ buffer has its
own address in every context, so each switch must make the library look the
buffer's address up again.  Device memory for the inputs and outputs comes
from the driver (cuMemAlloc) in the context current at the time.  Each result
is checked element by element against the fp64 oracle.  Prints "ok" and exits
0 on success; exits 1 with a message otherwise.
"""
import ctypes
import math
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from exact_attention_127_b200 import inputs  # noqa: E402

O_MAX_ABS, O_REL_L2, LSE_MAX_ABS = 2e-2, 5e-3, 1e-3

cu = ctypes.CDLL("libcuda.so.1")
lib = ctypes.CDLL(os.path.join(ROOT, "exact_attention_127_b200", "libattn127.so"))
vp, i64 = ctypes.c_void_p, ctypes.c_int64
lib.attn_decode_noalloc.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i64, ctypes.c_float, vp]
lib.attn_decode_noalloc.restype = ctypes.c_int
lib.attn_device_status.argtypes = [vp, ctypes.c_int]
lib.attn_device_status.restype = ctypes.c_int


def check(rc, what):
    if rc != 0:
        sys.stderr.write(f"{what} failed with {rc}\n")
        sys.exit(1)


def bf16_bytes(t):
    return np.ascontiguousarray(t.contiguous().view(dtype=__import__("torch").int16).numpy())


def run_once(label, B, H, N, d, seed):
    q, k, v = inputs.make_decode_qkv(B, H, N, d, seed)
    host = [bf16_bytes(t) for t in (q, k, v)]
    ptrs = []
    for a in host:
        p = ctypes.c_uint64()
        check(cu.cuMemAlloc_v2(ctypes.byref(p), ctypes.c_size_t(a.nbytes)), "cuMemAlloc")
        check(cu.cuMemcpyHtoD_v2(p, a.ctypes.data_as(vp), ctypes.c_size_t(a.nbytes)), "cuMemcpyHtoD")
        ptrs.append(p)
    o = ctypes.c_uint64()
    lse = ctypes.c_uint64()
    check(cu.cuMemAlloc_v2(ctypes.byref(o), ctypes.c_size_t(B * H * d * 2)), "cuMemAlloc")
    check(cu.cuMemAlloc_v2(ctypes.byref(lse), ctypes.c_size_t(B * H * 4)), "cuMemAlloc")
    rc = lib.attn_decode_noalloc(ptrs[0].value, ptrs[1].value, ptrs[2].value, o.value, lse.value,
                                 B, H, N, d, 1.0 / math.sqrt(d), None)
    check(rc, f"{label}: attn_decode_noalloc")
    check(cu.cuCtxSynchronize(), f"{label}: cuCtxSynchronize")
    check(lib.attn_device_status(None, 1), f"{label}: device status")
    o_raw = np.empty(B * H * d, dtype=np.uint16)
    l_out = np.empty(B * H, dtype=np.float32)
    check(cu.cuMemcpyDtoH_v2(o_raw.ctypes.data_as(vp), o, ctypes.c_size_t(o_raw.nbytes)), "DtoH")
    check(cu.cuMemcpyDtoH_v2(l_out.ctypes.data_as(vp), lse, ctypes.c_size_t(l_out.nbytes)), "DtoH")
    for p in ptrs + [o, lse]:
        check(cu.cuMemFree_v2(p), "cuMemFree")
    o_f = (o_raw.astype(np.uint32) << 16).view(np.float32).astype(np.float64).reshape(B * H, 1, d)
    O, L = oracle.attention_qk(q, k, v, 1.0 / math.sqrt(d))
    err = np.abs(o_f - O).max()
    rel = np.linalg.norm(o_f - O) / np.linalg.norm(O)
    lerr = np.abs(l_out.astype(np.float64).reshape(B * H, 1) - L).max()
    if not (err <= O_MAX_ABS and rel <= O_REL_L2 and lerr <= LSE_MAX_ABS):
        sys.stderr.write(f"{label}: max|dO|={err:.3e} relL2={rel:.3e} max|dLSE|={lerr:.3e}\n")
        sys.exit(1)
    print(f"{label}: max|dO|={err:.3e} relL2={rel:.3e} max|dLSE|={lerr:.3e}")


def main():
    check(cu.cuInit(0), "cuInit")
    dev = ctypes.c_int()
    check(cu.cuDeviceGet(ctypes.byref(dev), 0), "cuDeviceGet")
    primary = ctypes.c_void_p()
    check(cu.cuDevicePrimaryCtxRetain(ctypes.byref(primary), dev), "cuDevicePrimaryCtxRetain")
    check(cu.cuCtxSetCurrent(primary), "cuCtxSetCurrent")
    run_once("primary context", 2, 3, 1500, 128, 51)
    second = ctypes.c_void_p()
    check(cu.cuCtxCreate_v2(ctypes.byref(second), 0, dev), "cuCtxCreate")   # now current
    run_once("second context", 1, 4, 700, 64, 52)
    check(cu.cuCtxSetCurrent(primary), "cuCtxSetCurrent")
    run_once("primary context again", 3, 2, 2100, 128, 53)
    check(cu.cuCtxDestroy_v2(second), "cuCtxDestroy")
    print("ok")


if __name__ == "__main__":
    main()
