"""Child process of the no-alloc test: the ring backward that allocates
nothing, before and after a device reset.

A device reset destroys the context that loaded the library's device code;
the next call loads it again, possibly at another address.  This script
drives the C ABI with the CUDA runtime alone (no torch device memory, whose
allocator would not survive the reset): it runs the ring forward, the no-alloc
backward and the workspace backward, resets the device, runs all three again
on freshly copied inputs, and exits 0 only if the four backward results are
bit-identical.  Run by tests/test_zz_no_alloc.py; not collected by pytest.
"""

import ctypes
import os
import sys

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from sequence_attention_rm_b200 import rm, synthetic  # noqa: E402


def _cudart() -> ctypes.CDLL:
    """The CUDA runtime librm_attn.so is linked against (already mapped)."""
    with open("/proc/self/maps") as f:
        for line in f:
            path = line.split()[-1]
            if "libcudart.so" in path:
                return ctypes.CDLL(path)
    return ctypes.CDLL("libcudart.so.12")


CUDART = _cudart()
H2D, D2H = 1, 2


def _ok(err, what):
    if err != 0:
        raise RuntimeError(f"{what}: cuda error {err}")


def _rm_ok(status, what):
    if status != rm.RM_OK:
        raise RuntimeError(f"{what}: {rm._lib.rm_last_error().decode()}")


class Dev:
    """Device buffers of one run, freed together."""

    def __init__(self):
        self.ptrs = []

    def alloc(self, nbytes):
        p = ctypes.c_void_p()
        _ok(CUDART.cudaMalloc(ctypes.byref(p), ctypes.c_size_t(max(nbytes, 256))), "cudaMalloc")
        self.ptrs.append(p)
        return p

    def upload(self, arr):
        arr = np.ascontiguousarray(arr)
        p = self.alloc(arr.nbytes)
        _ok(CUDART.cudaMemcpy(p, arr.ctypes.data_as(ctypes.c_void_p), ctypes.c_size_t(arr.nbytes),
                              H2D), "upload")
        return p

    def download(self, p, like):
        out = np.empty_like(like)
        _ok(CUDART.cudaMemcpy(out.ctypes.data_as(ctypes.c_void_p), p, ctypes.c_size_t(out.nbytes),
                              D2H), "download")
        return out

    def free(self):
        for p in self.ptrs:
            CUDART.cudaFree(p)
        self.ptrs = []


def run_once(w, host):
    """Forward, no-alloc backward, workspace backward; returns both results."""
    lib = rm._lib
    B, N, Hq, Hkv, d = w.B, w.N, w.Hq, w.Hkv, w.d
    dsc = rm.RmAttnDesc(rm.RM_BF16, B, Hq, Hkv, d, N, w.P, rm.LAYOUTS[w.layout], 1, 0.0,
                        rm.MODES["fused"], rm.ORDERS["rank"], None, 0, None)
    dev = Dev()
    try:
        q, k, v, do = (dev.upload(x) for x in host)
        o = dev.alloc(host[0].nbytes)
        lse = dev.alloc(B * Hq * N * 4)
        grads = [[dev.alloc(x.nbytes) for x in (host[0], host[1], host[2])] for _ in range(2)]
        ws_bytes = ctypes.c_size_t()
        _rm_ok(lib.rm_ring_workspace_size(ctypes.byref(dsc), 1, ctypes.byref(ws_bytes)), "ws size")
        ws = dev.alloc(ws_bytes.value)
        tq = lambda p: rm.RmTensor(p, N * Hq * d, Hq * d, d)
        tk = lambda p: rm.RmTensor(p, N * Hkv * d, Hkv * d, d)
        null = ctypes.c_void_p(0)
        _rm_ok(lib.rm_ring_attn_fwd(ctypes.byref(dsc), tq(q), tk(k), tk(v), tq(o), lse, null, 0,
                                    null), "ring fwd")
        (a_dq, a_dk, a_dv), (b_dq, b_dk, b_dv) = grads
        _rm_ok(lib.rm_ring_attn_bwd_noalloc(ctypes.byref(dsc), tq(q), tk(k), tk(v), tq(o), lse,
                                            tq(do), tq(a_dq), tk(a_dk), tk(a_dv), null),
               "no-alloc bwd")
        _rm_ok(lib.rm_ring_attn_bwd(ctypes.byref(dsc), tq(q), tk(k), tk(v), tq(o), lse, tq(do),
                                    tq(b_dq), tk(b_dk), tk(b_dv), ws, ws_bytes, null),
               "workspace bwd")
        _ok(CUDART.cudaDeviceSynchronize(), "sync")
        _rm_ok(lib.rm_get_device_status(null), "device status")
        like = (host[0], host[1], host[2])
        return ([dev.download(p, x) for p, x in zip(grads[0], like)],
                [dev.download(p, x) for p, x in zip(grads[1], like)])
    finally:
        dev.free()


def main():
    w = synthetic.Workload(907, "no-alloc-reset", B=1, Hq=4, Hkv=2, N=1024, d=128, P=2,
                           layout="zigzag", causal=True, dtype=torch.bfloat16, qkv_scale=0.5)
    host = [t.contiguous().view(torch.int16).numpy() for t in synthetic.attention_inputs(w)]
    _ok(CUDART.cudaSetDevice(0), "cudaSetDevice")
    noalloc_1, ws_1 = run_once(w, host)
    _ok(CUDART.cudaDeviceReset(), "cudaDeviceReset")
    noalloc_2, ws_2 = run_once(w, host)
    for name, a1, b1, a2, b2 in zip(("dq", "dk", "dv"), noalloc_1, ws_1, noalloc_2, ws_2):
        for tag, x in (("no-alloc before reset", a1), ("no-alloc after reset", a2),
                       ("workspace after reset", b2)):
            if not np.array_equal(x, b1):
                print(f"{name}: {tag} differs from the workspace backward before the reset")
                return 1
    print("no-alloc reset ok")
    return 0


if __name__ == "__main__":
    sys.exit(main())
