"""Packed and right-padded batches (ringmaster "Status": dense causal
sequences or globally right-padded batches; packing by global position
boundaries, whatever the context-parallel strategy), forward and backward,
against the oracle's segment-aware attention: the tensor-core ring, the fp32
SIMT ring, sequences of at most 16 tokens, USP and Mesh2D.  Padding rows must
come out empty: O = 0, LSE = -inf, zero gradients."""

import numpy as np
import pytest
import torch

from oracle import attention as oatt
from oracle import layouts as olay
from oracle import mesh2d as omesh
from oracle import usp as ousp
from sequence_attention_rm_b200 import synthetic
from tests._helpers import (BF16_LSE_TOL, BF16_O_TOL, F32_TOL, assert_f32_close, assert_grad_close,
                            assert_max_abs, gpu, np64)

pytestmark = gpu


@pytest.fixture(scope="module")
def rm():
    from sequence_attention_rm_b200 import rm as mod
    return mod


def _inputs(B, Hq, Hkv, N, d, seed, dtype=torch.bfloat16):
    w = synthetic.Workload(seed, "seg", B=B, Hq=Hq, Hkv=Hkv, N=N, d=d, P=1, layout="contiguous",
                           causal=True, dtype=dtype, qkv_scale=0.5 if dtype == torch.bfloat16 else 1.0)
    return synthetic.attention_inputs(w)


def _tols(dtype):
    return (F32_TOL, F32_TOL) if dtype == torch.float32 else (BF16_O_TOL, BF16_LSE_TOL)


def _grad_check(dtype):
    return assert_f32_close if dtype == torch.float32 else assert_grad_close


def _run(rm, q, k, v, do, *, P, layout, causal, order, mode="fused", d128=True, **segs):
    if order == "rank":
        perm = lambda x: rm.layout_permute(x, layout, P)
        back = lambda x: rm.layout_permute(x, layout, P, inverse=True)
    else:
        perm = back = lambda x: x
    qg, kg, vg, dog = (perm(t.cuda()) for t in (q, k, v, do))
    o, l = rm.ring_attn_fwd(qg, kg, vg, P=P, layout=layout, causal=causal, order=order, mode=mode,
                            **segs)
    B, Hq, N = l.shape
    if order == "rank":
        lg = rm.layout_permute(l.reshape(B * Hq, N, 1, 1).contiguous(), layout, P,
                               inverse=True).reshape(B, Hq, N)
    else:
        lg = l
    grads = None
    if d128:
        grads = [back(g) for g in rm.ring_attn_bwd(qg, kg, vg, o, l, dog, P=P, layout=layout,
                                                   causal=causal, order=order, **segs)]
    return back(o), lg, grads


CU = [0, 100, 357, 358, 900, 1000]  # N = 1024: positions 1000.. are padding


@pytest.mark.parametrize("layout,P,order,causal", [
    ("zigzag", 2, "global", True), ("zigzag", 2, "rank", True), ("striped", 4, "rank", True),
    ("contiguous", 2, "rank", False), ("striped", 2, "global", False)])
def test_packed(rm, layout, P, order, causal):
    N = 1024
    q, k, v, do = _inputs(1, 8, 4, N, 128, 41)
    seg = oatt.segments_from_boundaries(CU, N)
    o_ref, l_ref = oatt.attention_forward(np64(q), np64(k), np64(v), causal=causal, seg=seg)
    g_ref = oatt.attention_backward(np64(q), np64(k), np64(v), np64(do), causal=causal, seg=seg)
    cu = torch.tensor(CU, dtype=torch.int32, device="cuda")
    o, l, grads = _run(rm, q, k, v, do, P=P, layout=layout, causal=causal, order=order,
                       cu_seqlens=cu)
    assert_max_abs(np64(o), o_ref, BF16_O_TOL, "O")
    assert_max_abs(np64(l), l_ref, BF16_LSE_TOL, "LSE")
    assert torch.all(o[:, 1000:] == 0) and torch.all(torch.isneginf(l[:, :, 1000:]))
    for name, g, ref in zip(("dq", "dk", "dv"), grads, g_ref):
        assert_grad_close(np64(g), ref, what=name)
        assert torch.all(g[:, 1000:] == 0), name


@pytest.mark.parametrize("layout,P,order", [("striped", 2, "rank"), ("zigzag", 2, "global")])
def test_right_padded(rm, layout, P, order):
    N, lengths = 1024, [1024, 700, 1]
    q, k, v, do = _inputs(3, 4, 2, N, 128, 43)
    seg = oatt.segments_from_lengths(lengths, N)
    o_ref, l_ref = oatt.attention_forward(np64(q), np64(k), np64(v), causal=True, seg=seg)
    g_ref = oatt.attention_backward(np64(q), np64(k), np64(v), np64(do), causal=True, seg=seg)
    lens = torch.tensor(lengths, dtype=torch.int32, device="cuda")
    o, l, grads = _run(rm, q, k, v, do, P=P, layout=layout, causal=True, order=order, seq_lens=lens)
    assert_max_abs(np64(o), o_ref, BF16_O_TOL, "O")
    assert_max_abs(np64(l), l_ref, BF16_LSE_TOL, "LSE")
    for name, g, ref in zip(("dq", "dk", "dv"), grads, g_ref):
        assert_grad_close(np64(g), ref, what=name)
    assert torch.all(o[1, 700:] == 0) and torch.all(grads[0][2, 1:] == 0)


def test_packed_forward_small_head_dim_and_stepwise(rm):
    N = 1024
    q, k, v, do = _inputs(1, 4, 2, N, 64, 47)
    seg = oatt.segments_from_boundaries(CU, N)
    o_ref, l_ref = oatt.attention_forward(np64(q), np64(k), np64(v), causal=True, seg=seg)
    cu = torch.tensor(CU, dtype=torch.int32, device="cuda")
    for mode in ("fused", "stepwise"):
        o, l, _ = _run(rm, q, k, v, do, P=2, layout="zigzag", causal=True, order="rank", mode=mode,
                       d128=False, cu_seqlens=cu)
        assert_max_abs(np64(o), o_ref, BF16_O_TOL, f"O {mode}")
        assert_max_abs(np64(l), l_ref, BF16_LSE_TOL, f"LSE {mode}")


@pytest.mark.parametrize("kind", ["packed", "padded"])
@pytest.mark.parametrize("layout,P,mode", [("zigzag", 2, "fused"), ("striped", 4, "fused"),
                                           ("contiguous", 2, "stepwise")])
def test_fp32_simt_ring(rm, kind, layout, P, mode):
    """fp32 problems run on the SIMT kernels: segment masks there, 1e-5."""
    N = 256
    B = 1 if kind == "packed" else 2
    q, k, v, do = _inputs(B, 4, 2, N, 64, 51, torch.float32)
    if kind == "packed":
        cu_l = [0, 30, 31, 140, 250]
        seg = oatt.segments_from_boundaries(cu_l, N)
        segs = dict(cu_seqlens=torch.tensor(cu_l, dtype=torch.int32, device="cuda"))
    else:
        seg = oatt.segments_from_lengths([N, 77], N)
        segs = dict(seq_lens=torch.tensor([N, 77], dtype=torch.int32, device="cuda"))
    o_ref, l_ref = oatt.attention_forward(np64(q), np64(k), np64(v), causal=True, seg=seg)
    g_ref = oatt.attention_backward(np64(q), np64(k), np64(v), np64(do), causal=True, seg=seg)
    o, l, grads = _run(rm, q, k, v, do, P=P, layout=layout, causal=True, order="rank", mode=mode,
                       **segs)
    assert_max_abs(np64(o), o_ref, F32_TOL, "O")
    assert_max_abs(np64(l), l_ref, F32_TOL, "LSE")
    for name, g, ref in zip(("dq", "dk", "dv"), grads, g_ref):
        assert_f32_close(np64(g), ref, name)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_short_sequences_take_the_general_kernels(rm, dtype):
    """Sequences of at most 16 tokens with segments: the short-sequence
    kernels have no segment masks, so these calls run on the general
    (tensor-core or SIMT) kernels; results match the oracle."""
    N, d = 16, 64
    q, k, v, do = _inputs(3, 2, 2, N, d, 53, dtype)
    seg = oatt.segments_from_lengths([16, 9, 1], N)
    lens = torch.tensor([16, 9, 1], dtype=torch.int32, device="cuda")
    o_ref, l_ref = oatt.attention_forward(np64(q), np64(k), np64(v), causal=False, seg=seg)
    o, l = rm.ring_attn_fwd(q.cuda(), k.cuda(), v.cuda(), P=1, layout="contiguous", causal=False,
                            seq_lens=lens)
    to, tl = _tols(dtype)
    assert_max_abs(np64(o), o_ref, to, "O")
    assert_max_abs(np64(l), l_ref, tl, "LSE")
    assert torch.all(o[2, 1:] == 0) and torch.all(torch.isneginf(l[2, :, 1:]))


USP_CASES = [
    # dtype, kind, layout, P (ring), U (ulysses), order
    (torch.bfloat16, "packed", "zigzag", 2, 2, "global"),
    (torch.bfloat16, "padded", "striped", 2, 2, "rank"),
    (torch.bfloat16, "packed", "contiguous", 1, 4, "rank"),
    (torch.float32, "packed", "zigzag", 2, 2, "rank"),
    (torch.float32, "padded", "contiguous", 2, 2, "rank"),
]


@pytest.mark.parametrize("case", USP_CASES, ids=lambda c: f"{str(c[0])[6:]}-{c[1]}-{c[2]}-P{c[3]}xU{c[4]}-{c[5]}")
def test_usp_with_segments(rm, case):
    dtype, kind, layout, P, U, order = case
    N = 512 if dtype == torch.bfloat16 else 128
    d = 128 if dtype == torch.bfloat16 else 64
    B = 1 if kind == "packed" else 2
    q, k, v, do = _inputs(B, 8, 4, N, d, 55 + N, dtype)
    if kind == "packed":
        cu_l = [0, 3, 64, 65, N - 40]
        seg = oatt.segments_from_boundaries(cu_l, N)
        segs = dict(cu_seqlens=torch.tensor(cu_l, dtype=torch.int32, device="cuda"))
    else:
        seg = oatt.segments_from_lengths([N, N // 3], N)
        segs = dict(seq_lens=torch.tensor([N, N // 3], dtype=torch.int32, device="cuda"))
    if order == "rank":
        perm = lambda x: olay.permute(np64(x), layout, P)
        o_ref, l_ref = ousp.usp_forward(perm(q), perm(k), perm(v), layout, P, U, True, seg=seg)
        g_ref = ousp.usp_backward(perm(q), perm(k), perm(v), o_ref, l_ref, perm(do), layout, P, U,
                                  True, seg=seg)
        gperm = lambda x: rm.layout_permute(x.cuda(), layout, P)
    else:  # global order: the definition itself
        o_ref, l_ref = oatt.attention_forward(np64(q), np64(k), np64(v), causal=True, seg=seg)
        g_ref = oatt.attention_backward(np64(q), np64(k), np64(v), np64(do), causal=True, seg=seg)
        gperm = lambda x: x.cuda()
    qg, kg, vg, dog = gperm(q), gperm(k), gperm(v), gperm(do)
    o, l = rm.usp_attn_fwd(qg, kg, vg, P=P, ulysses=U, layout=layout, causal=True, order=order,
                           **segs)
    to, tl = _tols(dtype)
    assert_max_abs(np64(o), o_ref, to, "O")
    assert_max_abs(np64(l), l_ref, tl, "LSE")
    grads = rm.usp_attn_bwd(qg, kg, vg, o, l, dog, P=P, ulysses=U, layout=layout, causal=True,
                            order=order, **segs)
    check = _grad_check(dtype)
    for name, g, ref in zip(("dq", "dk", "dv"), grads, g_ref):
        check(np64(g), ref, what=name)


MESH_CASES = [
    # dtype, kind, N, grid_q, grid_k, causal
    (torch.bfloat16, "packed", 1024, 2, 2, True),
    (torch.bfloat16, "padded", 768, 4, 2, True),
    (torch.bfloat16, "packed", 768, 2, 3, False),
    (torch.float32, "packed", 192, 3, 2, True),
    (torch.float32, "padded", 128, 2, 4, False),
]


@pytest.mark.parametrize("case", MESH_CASES, ids=lambda c: f"{str(c[0])[6:]}-{c[1]}-N{c[2]}-{c[3]}x{c[4]}-{'causal' if c[5] else 'full'}")
def test_mesh2d_with_segments(rm, case):
    dtype, kind, N, gq, gk, causal = case
    d = 128 if dtype == torch.bfloat16 else 64
    B = 1 if kind == "packed" else 2
    q, k, v, do = _inputs(B, 4, 2, N, d, 57 + N, dtype)
    if kind == "packed":
        cu_l = [0, 17, N // 2 + 5, N // 2 + 6, N - 20]
        seg = oatt.segments_from_boundaries(cu_l, N)
        segs = dict(cu_seqlens=torch.tensor(cu_l, dtype=torch.int32, device="cuda"))
    else:
        seg = oatt.segments_from_lengths([N - 1, N // 4], N)
        segs = dict(seq_lens=torch.tensor([N - 1, N // 4], dtype=torch.int32, device="cuda"))
    o_ref, l_ref = omesh.mesh2d_forward(np64(q), np64(k), np64(v), gq, gk, causal, seg=seg)
    g_ref = omesh.mesh2d_backward(np64(q), np64(k), np64(v), o_ref, l_ref, np64(do), gq, gk, causal,
                                  seg=seg)
    qg, kg, vg, dog = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    o, l = rm.mesh2d_attn_fwd(qg, kg, vg, grid_q=gq, grid_k=gk, causal=causal, **segs)
    to, tl = _tols(dtype)
    assert_max_abs(np64(o), o_ref, to, "O")
    assert_max_abs(np64(l), l_ref, tl, "LSE")
    grads = rm.mesh2d_attn_bwd(qg, kg, vg, o, l, dog, grid_q=gq, grid_k=gk, causal=causal, **segs)
    check = _grad_check(dtype)
    for name, g, ref in zip(("dq", "dk", "dv"), grads, g_ref):
        check(np64(g), ref, what=name)
