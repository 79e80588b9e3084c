"""The ring backward that allocates nothing (rm_ring_attn_bwd_noalloc).

Some callers cannot allocate device memory: a runtime that reserved all of it
for its own pool, or code that must not call cudaMalloc because it would
synchronise the device.  This entry point runs the ring backward out of a
fixed 64 MiB scratch array inside the library instead of a caller-provided
workspace.  The backward is deterministic and both entry points run the same
kernels, so their results must be bit-identical, call after call: the scratch
keeps the previous call's contents, which must not leak into the next result.
The first call here is the larger problem, so the second finds stale values
beyond the part of the scratch it writes.  This file is collected last so that
a run stopping at its first failure has already run every other test.
"""

import ctypes
import os
import subprocess
import sys

import pytest
import torch

from sequence_attention_rm_b200 import synthetic
from tests._helpers import gpu

pytestmark = gpu

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.fixture(scope="module")
def rm():
    from sequence_attention_rm_b200 import rm as mod
    return mod


def _problem(rm, seed, Hq, Hkv, N):
    w = synthetic.Workload(seed, "no-alloc", B=1, Hq=Hq, Hkv=Hkv, N=N, d=128, P=2,
                           layout="zigzag", causal=True, dtype=torch.bfloat16, qkv_scale=0.5)
    q, k, v, do = (t.cuda() for t in synthetic.attention_inputs(w))
    perm = lambda x: rm.layout_permute(x, w.layout, w.P)
    qr, kr, vr, dor = perm(q), perm(k), perm(v), perm(do)
    o, lse = rm.ring_attn_fwd(qr, kr, vr, P=w.P, layout=w.layout, causal=True)
    return w, qr, kr, vr, dor, o, lse


def test_no_alloc_backward_matches_the_workspace_backward(rm):
    lib = rm.raw()
    # two calls in a row, different inputs; the first one is the larger, so it
    # leaves scratch contents past the end of what the second one writes
    for call, (seed, Hq, Hkv, N) in enumerate(((901, 8, 4, 4096), (902, 4, 2, 2048))):
        w, qr, kr, vr, dor, o, lse = _problem(rm, seed, Hq, Hkv, N)
        ref = rm.ring_attn_bwd(qr, kr, vr, o, lse, dor, P=w.P, layout=w.layout, causal=True)
        dsc = rm.desc(w.dtype, w.B, w.Hq, w.Hkv, w.d, w.N, w.P, w.layout, True)
        dq, dk, dv = torch.empty_like(qr), torch.empty_like(kr), torch.empty_like(vr)
        st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
        status = lib.rm_ring_attn_bwd_noalloc(
            ctypes.byref(dsc), rm._bnhd(qr), rm._bnhd(kr), rm._bnhd(vr), rm._bnhd(o),
            ctypes.c_void_p(lse.data_ptr()), rm._bnhd(dor), rm._bnhd(dq), rm._bnhd(dk),
            rm._bnhd(dv), st)
        assert status == rm.RM_OK, lib.rm_last_error()
        torch.cuda.synchronize()
        assert rm.get_device_status() == rm.RM_OK
        for name, got, want in zip(("dq", "dk", "dv"), (dq, dk, dv), ref):
            assert torch.equal(got, want), f"call {call} {name}: differs from rm_ring_attn_bwd"


def test_no_alloc_rejects_problems_beyond_its_scratch(rm):
    lib = rm.raw()
    # workspace = delta [B, Hq, N] fp32 = 16 * 2^21 * 4 bytes = 128 MiB > 64 MiB
    n = 1 << 21
    dsc = rm.desc(torch.bfloat16, 1, 16, 8, 128, n, 2, "zigzag", True)
    assert rm.ring_workspace_size(dsc, True) > 64 << 20
    T = rm.RmTensor
    x = torch.empty(16, device="cuda")
    t = T(x.data_ptr(), n * 16 * 128, 16 * 128, 128)
    nul = ctypes.c_void_p(0)
    status = lib.rm_ring_attn_bwd_noalloc(ctypes.byref(dsc), t, t, t, t, nul, t, t, t, t, nul)
    assert status == rm.RM_ERR_WORKSPACE
    assert b"64" in lib.rm_last_error() or b"scratch" in lib.rm_last_error()


def test_no_alloc_survives_a_device_reset():
    """A device reset ends the context that loaded the scratch array; the next
    call must find the array in the new context.  Run in a child process that
    holds no torch device memory (torch's allocator would not survive the
    reset)."""
    res = subprocess.run([sys.executable, os.path.join(HERE, "noalloc_reset_child.py")],
                         capture_output=True, text=True, timeout=600)
    assert res.returncode == 0, res.stdout[-2000:] + res.stderr[-2000:]
    assert "no-alloc reset ok" in res.stdout
