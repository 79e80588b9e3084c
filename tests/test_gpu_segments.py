"""Packed and right-padded batches on the tensor-core ring (ringmaster
"Status": dense causal sequences or globally right-padded batches; packing
by global position boundaries), forward and backward, against the oracle's
segment-aware attention.  Padding rows must come out empty: O = 0,
LSE = -inf, zero gradients."""

import numpy as np
import pytest
import torch

from oracle import attention as oatt
from sequence_attention_rm_b200 import synthetic
from tests._helpers import BF16_LSE_TOL, BF16_O_TOL, assert_grad_close, assert_max_abs, gpu, np64

pytestmark = gpu


@pytest.fixture(scope="module")
def rm():
    from sequence_attention_rm_b200 import rm as mod
    return mod


def _inputs(B, Hq, Hkv, N, d, seed):
    w = synthetic.Workload(seed, "seg", B=B, Hq=Hq, Hkv=Hkv, N=N, d=d, P=1, layout="contiguous",
                           causal=True, dtype=torch.bfloat16, qkv_scale=0.5)
    return synthetic.attention_inputs(w)


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


def test_segments_rejected_for_fp32(rm):
    q = torch.zeros(1, 64, 2, 64, device="cuda")
    cu = torch.tensor([0, 10, 64], dtype=torch.int32, device="cuda")
    with pytest.raises(rm.RmError):
        rm.ring_attn_fwd(q, q, q, P=2, layout="contiguous", causal=True, cu_seqlens=cu)
