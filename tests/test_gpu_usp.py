"""USP on one GPU (ringmaster "Why": Ulysses x ring on a 2-D mesh): the
library's repack -> ring -> repack composition against the oracle's, forward
and backward, rank-major and global token order, bf16 and fp32."""

import numpy as np
import pytest
import torch

from oracle import attention as oatt
from oracle import layouts as olay
from oracle import usp as ousp
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
    w = synthetic.Workload(seed, "usp", B=B, Hq=Hq, Hkv=Hkv, N=N, d=d, P=1, layout="contiguous",
                           causal=True, dtype=dtype, qkv_scale=0.5 if dtype == torch.bfloat16 else 1.0)
    return synthetic.attention_inputs(w)


CASES = [
    # dtype, B, Hq, Hkv, N, d, P(ring), ulysses, layout, causal
    (torch.bfloat16, 1, 16, 8, 1024, 128, 2, 2, "zigzag", True),
    (torch.bfloat16, 2, 8, 4, 768, 128, 2, 4, "striped", True),
    (torch.bfloat16, 1, 4, 4, 512, 128, 1, 4, "contiguous", False),
    (torch.bfloat16, 1, 8, 2, 1040, 64, 4, 2, "striped", True),   # d = 64: backward on the SIMT kernels
    (torch.float32, 1, 4, 2, 128, 64, 2, 2, "contiguous", True),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"{str(c[0])[6:]}-B{c[1]}H{c[2]}/{c[3]}-N{c[4]}-d{c[5]}-P{c[6]}xU{c[7]}-{c[8]}")
def test_usp_matches_oracle(rm, case):
    dtype, B, Hq, Hkv, N, d, P, U, layout, causal = case
    q, k, v, do = _inputs(dtype, B, Hq, Hkv, N, d, 60 + N)
    perm = lambda x: olay.permute(np64(x), layout, P)
    o_ref, l_ref = ousp.usp_forward(perm(q), perm(k), perm(v), layout, P, U, causal)
    gperm = lambda x: rm.layout_permute(x.cuda(), layout, P)
    qg, kg, vg, dog = gperm(q), gperm(k), gperm(v), gperm(do)
    o, l = rm.usp_attn_fwd(qg, kg, vg, P=P, ulysses=U, layout=layout, causal=causal)
    tol_o, tol_l = (F32_TOL, F32_TOL) if dtype == torch.float32 else (BF16_O_TOL, BF16_LSE_TOL)
    assert_max_abs(np64(o), o_ref, tol_o, "O")
    assert_max_abs(np64(l), l_ref, tol_l, "LSE")
    g_ref = ousp.usp_backward(perm(q), perm(k), perm(v), o_ref, l_ref, perm(do), layout, P, U,
                              causal)
    grads = rm.usp_attn_bwd(qg, kg, vg, o, l, dog, P=P, ulysses=U, layout=layout, causal=causal)
    for name, g, ref in zip(("dq", "dk", "dv"), grads, g_ref):
        if dtype == torch.float32:
            assert_f32_close(np64(g), ref, name)
        else:
            assert_grad_close(np64(g), ref, what=name)


def test_usp_global_order_is_plain_attention(rm):
    """Global-order operands straight against the definition (no permutes)."""
    q, k, v, do = _inputs(torch.bfloat16, 1, 8, 4, 1024, 128, 99)
    o_ref, l_ref = oatt.attention_forward(np64(q), np64(k), np64(v), causal=True)
    g_ref = oatt.attention_backward(np64(q), np64(k), np64(v), np64(do), causal=True)
    qg, kg, vg, dog = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    o, l = rm.usp_attn_fwd(qg, kg, vg, P=2, ulysses=2, layout="zigzag", causal=True, order="global")
    assert_max_abs(np64(o), o_ref, BF16_O_TOL, "O")
    assert_max_abs(np64(l), l_ref, BF16_LSE_TOL, "LSE")
    grads = rm.usp_attn_bwd(qg, kg, vg, o, l, dog, P=2, ulysses=2, layout="zigzag", causal=True,
                            order="global")
    for name, g, ref in zip(("dq", "dk", "dv"), grads, g_ref):
        assert_grad_close(np64(g), ref, what=name)


def test_usp_rejects_bad_degree(rm):
    q = torch.zeros(1, 256, 8, 128, dtype=torch.bfloat16, device="cuda")
    k = torch.zeros(1, 256, 4, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(rm.RmError):
        rm.usp_attn_fwd(q, k, k, P=2, ulysses=8, layout="zigzag", causal=True)  # 8 > Hkv
    with pytest.raises(rm.RmError):
        rm.usp_attn_fwd(q, k, k, P=2, ulysses=3, layout="zigzag", causal=True)  # 3 does not divide
