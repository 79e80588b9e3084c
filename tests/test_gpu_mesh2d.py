"""Mesh2D on one GPU (Mosaic page, "Beyond 1D: Mesh2D Attention"): the
library's grid of (query chunk, key chunk) tiles, merged per query chunk,
against the oracle's, forward and backward, square and rectangular grids,
ragged chunks, bf16 and fp32."""

import ctypes

import pytest
import torch

from oracle import mesh2d as omesh
from sequence_attention_rm_b200 import synthetic
from tests._helpers import (BF16_LSE_TOL, BF16_O_TOL, F32_TOL, assert_f32_close, assert_grad_close,
                            assert_max_abs,
                            gpu, np64)

pytestmark = gpu


@pytest.fixture(scope="module")
def rm():
    from sequence_attention_rm_b200 import rm as mod
    return mod


def _inputs(dtype, B, Hq, Hkv, N, d, seed):
    w = synthetic.Workload(seed, "mesh2d", B=B, Hq=Hq, Hkv=Hkv, N=N, d=d, P=1,
                           layout="contiguous", causal=True, dtype=dtype,
                           qkv_scale=0.5 if dtype == torch.bfloat16 else 1.0)
    return synthetic.attention_inputs(w)


CASES = [
    # dtype, B, Hq, Hkv, N, d, grid_q, grid_k, causal
    (torch.bfloat16, 1, 8, 4, 1024, 128, 2, 2, True),
    (torch.bfloat16, 1, 8, 4, 1024, 128, 4, 4, True),
    (torch.bfloat16, 2, 4, 2, 768, 128, 2, 4, True),     # rectangular: chunks 384 / 192
    (torch.bfloat16, 1, 4, 4, 768, 128, 4, 2, False),
    (torch.bfloat16, 1, 4, 2, 600, 128, 2, 3, True),     # ragged chunks 300 / 200
    (torch.bfloat16, 1, 4, 2, 1200, 128, 3, 8, True),    # chunks 400 / 150
    (torch.bfloat16, 1, 8, 2, 640, 64, 5, 2, True),      # d = 64: backward on the SIMT kernels
    (torch.float32, 1, 4, 2, 384, 64, 2, 3, True),
    (torch.float32, 2, 2, 2, 96, 32, 3, 4, False),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"{str(c[0])[6:]}-B{c[1]}H{c[2]}/{c[3]}-N{c[4]}-d{c[5]}-{c[6]}x{c[7]}-{'causal' if c[8] else 'full'}")
def test_mesh2d_matches_oracle(rm, case):
    dtype, B, Hq, Hkv, N, d, gq, gk, causal = case
    q, k, v, do = _inputs(dtype, B, Hq, Hkv, N, d, 90 + N + gq * 16 + gk)
    o_ref, l_ref = omesh.mesh2d_forward(np64(q), np64(k), np64(v), gq, gk, causal)
    qg, kg, vg, dog = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    o, l = rm.mesh2d_attn_fwd(qg, kg, vg, grid_q=gq, grid_k=gk, causal=causal)
    tol_o, tol_l = (F32_TOL, F32_TOL) if dtype == torch.float32 else (BF16_O_TOL, BF16_LSE_TOL)
    assert_max_abs(np64(o), o_ref, tol_o, "O")
    assert_max_abs(np64(l), l_ref, tol_l, "LSE")
    g_ref = omesh.mesh2d_backward(np64(q), np64(k), np64(v), o_ref, l_ref, np64(do), gq, gk,
                                  causal)
    grads = rm.mesh2d_attn_bwd(qg, kg, vg, o, l, dog, grid_q=gq, grid_k=gk, causal=causal)
    for name, g, ref in zip(("dq", "dk", "dv"), grads, g_ref):
        assert g.dtype == dtype
        if dtype == torch.float32:
            assert_f32_close(np64(g), ref, name)
        else:
            assert_grad_close(np64(g), ref, what=name)


def test_mesh2d_strided_operands(rm):
    """q / k / v as views of packed qkv tensors, o into a strided view."""
    B, N, Hq, Hkv, d = 1, 512, 4, 2, 128
    q, k, v, do = _inputs(torch.bfloat16, B, Hq, Hkv, N, d, 7)
    kv = torch.cat([k, v], dim=2).cuda()  # [B, N, 2 Hkv, d]
    out = torch.empty(B, N, Hq + 1, d, dtype=torch.bfloat16, device="cuda")
    o, l = rm.mesh2d_attn_fwd(q.cuda(), kv[:, :, :Hkv], kv[:, :, Hkv:], grid_q=2, grid_k=2,
                              causal=True, out=out[:, :, :Hq])
    o_ref, l_ref = omesh.mesh2d_forward(np64(q), np64(k), np64(v), 2, 2, True)
    assert_max_abs(np64(o), o_ref, BF16_O_TOL, "O")
    assert_max_abs(np64(l), l_ref, BF16_LSE_TOL, "LSE")


def test_mesh2d_rejects_bad_grids(rm):
    q = torch.zeros(1, 64, 2, 64, device="cuda", dtype=torch.bfloat16)
    with pytest.raises(rm.RmError):
        rm.mesh2d_attn_fwd(q, q, q, grid_q=3, grid_k=1, causal=True)
    with pytest.raises(rm.RmError):
        rm.mesh2d_attn_fwd(q, q, q, grid_q=2, grid_k=32, causal=True)
    # packed batches need B == 1, as for the ring
    cu = torch.tensor([0, 10, 64], dtype=torch.int32, device="cuda")
    dsc = rm.desc(torch.bfloat16, 1, 2, 2, 64, 64, 2, "contiguous", True, cu_seqlens=cu)
    dsc.B = 2
    n = ctypes.c_size_t(0)
    assert rm.raw().rm_mesh2d_workspace_size(ctypes.byref(dsc), 2, 2, 0, ctypes.byref(n)) == 1
