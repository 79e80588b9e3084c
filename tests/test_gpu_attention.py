"""GPU parity of the attention path (block and ring, forward and backward)
against the fp64 oracle at sizes that span several tiles and a ragged tail.

fp32 problems run on the exact-fp32 SIMT kernels (tolerance 1e-5); bf16
problems run on the tcgen05 tensor-core kernels (O 2e-2, LSE 1e-3)."""

import numpy as np
import pytest
import torch

from oracle import attention as oatt
from oracle import layouts as olay
from oracle import ring as oring
from sequence_attention_rm_b200 import synthetic
from tests._helpers import (BF16_LSE_TOL, BF16_O_TOL, F32_TOL, assert_grad_close, assert_max_abs,
                            gpu, np64)

pytestmark = gpu


@pytest.fixture(scope="module")
def rm():
    from sequence_attention_rm_b200 import rm as mod
    return mod


def _tols(dtype):
    return (F32_TOL, F32_TOL) if dtype == torch.float32 else (BF16_O_TOL, BF16_LSE_TOL)


def _plain(q, k, v, causal):
    return oatt.attention_forward(np64(q), np64(k), np64(v), causal=causal)


def test_tiny_noncausal_ring_fp32_full(rm):
    """The tiny fp32 workload in full: H=2, N=256, d=64, P=4 contiguous."""
    w = synthetic.TINY_RING
    q, k, v, _ = synthetic.attention_inputs(w, with_dout=False)
    o_ref, l_ref = _plain(q, k, v, False)
    for mode in ("fused", "stepwise"):
        o, l = rm.ring_attn_fwd(q.cuda(), k.cuda(), v.cuda(), P=4, layout="contiguous",
                                causal=False, mode=mode)
        assert_max_abs(np64(o), o_ref, F32_TOL, f"O {mode}")
        assert_max_abs(np64(l), l_ref, F32_TOL, f"LSE {mode}")


CASES = [
    # dtype, B, Hq, Hkv, N, d, P, layout, causal
    (torch.float32, 1, 2, 2, 256, 64, 4, "contiguous", True),
    (torch.float32, 2, 4, 2, 200, 32, 2, "zigzag", True),
    (torch.float32, 1, 3, 1, 96, 128, 8, "striped", True),
    (torch.bfloat16, 1, 16, 8, 1024, 128, 2, "zigzag", True),
    (torch.bfloat16, 1, 4, 2, 1000, 128, 2, "zigzag", True),
    (torch.bfloat16, 1, 4, 2, 1040, 128, 8, "striped", True),
    (torch.bfloat16, 2, 4, 2, 768, 128, 4, "contiguous", True),
    (torch.bfloat16, 1, 4, 2, 2048, 128, 8, "zigzag", False),
    (torch.bfloat16, 1, 4, 2, 2048, 128, 4, "zigzag", True),
    (torch.bfloat16, 1, 3, 3, 600, 64, 2, "zigzag", True),
    (torch.bfloat16, 1, 2, 1, 520, 64, 4, "striped", True),
    (torch.bfloat16, 1, 4, 4, 800, 32, 2, "contiguous", True),
]


def _inputs(dtype, B, Hq, Hkv, N, d, seed):
    w = synthetic.Workload(seed, "case", B=B, Hq=Hq, Hkv=Hkv, N=N, d=d, P=1, layout="contiguous",
                           causal=True, dtype=dtype, qkv_scale=0.5 if dtype == torch.bfloat16 else 1.0)
    return synthetic.attention_inputs(w)


@pytest.mark.parametrize("mode", ["fused", "stepwise"])
@pytest.mark.parametrize("case", CASES, ids=lambda c: f"{str(c[0])[6:]}-B{c[1]}H{c[2]}/{c[3]}-N{c[4]}-d{c[5]}-P{c[6]}-{c[7]}-{'c' if c[8] else 'nc'}")
def test_ring_forward(rm, case, mode):
    dtype, B, Hq, Hkv, N, d, P, layout, causal = case
    q, k, v, _ = _inputs(dtype, B, Hq, Hkv, N, d, 50 + N + d)
    o_ref, l_ref = _plain(q, k, v, causal)          # plain attention, global order
    perm = lambda x: rm.layout_permute(x.cuda(), layout, P)
    o, l = rm.ring_attn_fwd(perm(q), perm(k), perm(v), P=P, layout=layout, causal=causal, mode=mode)
    o_g = rm.layout_permute(o, layout, P, inverse=True)
    l_g = olay.unpermute(np64(l), layout, P, axis=2)
    to, tl = _tols(dtype)
    assert_max_abs(np64(o_g), o_ref, to, "O")
    assert_max_abs(l_g, l_ref, tl, "LSE")


@pytest.mark.parametrize("case", [CASES[1], CASES[4], CASES[8], CASES[10]],
                         ids=["f32", "bf16-d128", "bf16-d64", "bf16-d32"])
def test_block_forward_every_pair(rm, case):
    dtype, B, Hq, Hkv, N, d, P, layout, causal = case
    q, k, v, _ = _inputs(dtype, B, Hq, Hkv, N, d, 70 + N)
    qr, kr, vr = (olay.permute(np64(x), layout, P) for x in (q, k, v))
    L = N // P
    dq = lambda x: torch.from_numpy(olay.permute(x.float().numpy(), layout, P)).to(dtype).cuda()
    qg, kg, vg = dq(q), dq(k), dq(v)
    to, tl = _tols(dtype)
    for r in range(P):
        for s in range(P):
            o, l = rm.attn_block_fwd(qg[:, r * L:(r + 1) * L], kg[:, s * L:(s + 1) * L],
                                     vg[:, s * L:(s + 1) * L], N=N, P=P, layout=layout,
                                     causal=causal, q_rank=r, kv_rank=s, o_f32=True)
            o_ref, l_ref = oatt.attention_forward(
                qr[:, r * L:(r + 1) * L], kr[:, s * L:(s + 1) * L], vr[:, s * L:(s + 1) * L],
                causal=causal, q_pos=olay.rank_positions(layout, N, P, r),
                k_pos=olay.rank_positions(layout, N, P, s))
            assert_max_abs(np64(o), o_ref, to, f"O pair ({r},{s})")
            assert_max_abs(np64(l), l_ref, tl, f"LSE pair ({r},{s})")


def test_block_forward_fully_masked_pair(rm):
    # contiguous causal: rank 0's queries see nothing of rank 1's keys
    q, k, v, _ = _inputs(torch.bfloat16, 1, 2, 1, 512, 128, 3)
    o, l = rm.attn_block_fwd(q[:, :256].cuda(), k[:, 256:].cuda(), v[:, 256:].cuda(), N=512, P=2,
                             layout="contiguous", causal=True, q_rank=0, kv_rank=1)
    assert torch.all(o == 0) and torch.all(torch.isneginf(l))


@pytest.mark.parametrize("case", [CASES[0], CASES[1], CASES[2]], ids=["contig", "zigzag", "striped"])
def test_ring_backward_fp32(rm, case):
    dtype, B, Hq, Hkv, N, d, P, layout, causal = case
    q, k, v, do = _inputs(dtype, B, Hq, Hkv, N, d, 90 + N)
    g_ref = oatt.attention_backward(np64(q), np64(k), np64(v), np64(do), causal=causal)
    perm = lambda x: rm.layout_permute(x.cuda(), layout, P)
    qg, kg, vg, dog = perm(q), perm(k), perm(v), perm(do)
    o, l = rm.ring_attn_fwd(qg, kg, vg, P=P, layout=layout, causal=causal)
    grads = rm.ring_attn_bwd(qg, kg, vg, o, l, dog, P=P, layout=layout, causal=causal)
    for name, g, ref in zip(("dq", "dk", "dv"), grads, g_ref):
        assert_max_abs(np64(rm.layout_permute(g, layout, P, inverse=True)), ref, 1e-5 * max(1, np.abs(ref).max()), name)


def test_block_backward_fp32_accumulates(rm):
    dtype, B, Hq, Hkv, N, d, P, layout, causal = CASES[1]
    q, k, v, do = _inputs(dtype, B, Hq, Hkv, N, d, 123)
    qr, kr, vr, dor = (olay.permute(np64(x), layout, P) for x in (q, k, v, do))
    o_ref, l_ref = oring.ring_forward(qr, kr, vr, layout, P, causal)
    g_ref = oring.ring_backward(qr, kr, vr, o_ref, l_ref, dor, layout, P, causal)
    L = N // P
    t = lambda x: torch.from_numpy(np.ascontiguousarray(x)).float().cuda()
    qg, kg, vg, dog = t(qr), t(kr), t(vr), t(dor)
    lse = t(l_ref)
    delta = t(oatt.delta_from_output(dor, o_ref))
    dq = torch.zeros_like(qg); dk = torch.zeros_like(kg); dv = torch.zeros_like(vg)
    for r in range(P):
        rows = slice(r * L, (r + 1) * L)
        for s in range(P):
            cols = slice(s * L, (s + 1) * L)
            rm.attn_block_bwd(qg[:, rows], kg[:, cols], vg[:, cols], dog[:, rows],
                              lse[:, :, rows].contiguous(), delta[:, :, rows].contiguous(),
                              dq[:, rows], dk[:, cols], dv[:, cols], N=N, P=P, layout=layout,
                              causal=causal, q_rank=r, kv_rank=s)
    for name, g, ref in zip(("dq", "dk", "dv"), (dq, dk, dv), g_ref):
        assert_max_abs(np64(g), ref, 1e-5 * max(1, np.abs(ref).max()), name)


BWD_CASES = [c for c in CASES if c[0] == torch.bfloat16 and c[5] == 128]


@pytest.mark.parametrize("case", BWD_CASES, ids=lambda c: f"B{c[1]}H{c[2]}/{c[3]}-N{c[4]}-P{c[6]}-{c[7]}-{'c' if c[8] else 'nc'}")
def test_ring_backward_bf16(rm, case):
    dtype, B, Hq, Hkv, N, d, P, layout, causal = case
    q, k, v, do = _inputs(dtype, B, Hq, Hkv, N, d, 190 + N)
    g_ref = oatt.attention_backward(np64(q), np64(k), np64(v), np64(do), causal=causal)
    perm = lambda x: rm.layout_permute(x.cuda(), layout, P)
    qg, kg, vg, dog = perm(q), perm(k), perm(v), perm(do)
    o, l = rm.ring_attn_fwd(qg, kg, vg, P=P, layout=layout, causal=causal)
    grads = rm.ring_attn_bwd(qg, kg, vg, o, l, dog, P=P, layout=layout, causal=causal)
    for name, g, ref in zip(("dq", "dk", "dv"), grads, g_ref):
        assert g.dtype == torch.bfloat16
        assert_grad_close(np64(rm.layout_permute(g, layout, P, inverse=True)), ref, what=name)


def test_block_backward_bf16_every_pair(rm):
    dtype, B, Hq, Hkv, N, d, P, layout, causal = CASES[4]
    q, k, v, do = _inputs(dtype, B, Hq, Hkv, N, d, 321)
    qr, kr, vr, dor = (olay.permute(np64(x), layout, P) for x in (q, k, v, do))
    o_ref, l_ref = oring.ring_forward(qr, kr, vr, layout, P, causal)
    g_ref = oring.ring_backward(qr, kr, vr, o_ref, l_ref, dor, layout, P, causal)
    L = N // P
    tb = lambda x: torch.from_numpy(np.ascontiguousarray(x)).to(torch.bfloat16).cuda()
    tf = lambda x: torch.from_numpy(np.ascontiguousarray(x)).float().cuda()
    qg, kg, vg, dog = tb(qr), tb(kr), tb(vr), tb(dor)
    lse, delta = tf(l_ref), tf(oatt.delta_from_output(dor, o_ref))
    dq = torch.zeros(qg.shape, dtype=torch.float32, device="cuda")
    dk = torch.zeros(kg.shape, dtype=torch.float32, device="cuda")
    dv = torch.zeros(vg.shape, dtype=torch.float32, device="cuda")
    for r in range(P):
        rows = slice(r * L, (r + 1) * L)
        for s in range(P):
            cols = slice(s * L, (s + 1) * L)
            rm.attn_block_bwd(qg[:, rows], kg[:, cols], vg[:, cols], dog[:, rows],
                              lse[:, :, rows].contiguous(), delta[:, :, rows].contiguous(),
                              dq[:, rows], dk[:, cols], dv[:, cols], N=N, P=P, layout=layout,
                              causal=causal, q_rank=r, kv_rank=s)
    for name, g, ref in zip(("dq", "dk", "dv"), (dq, dk, dv), g_ref):
        assert_grad_close(np64(g), ref, what=name)


@pytest.mark.parametrize("d", [64, 32, 24])
@pytest.mark.parametrize("layout,P", [("zigzag", 2), ("striped", 4), ("contiguous", 2)])
def test_bf16_backward_other_head_dims(rm, d, layout, P):
    """bf16 at head dims other than 128: the backward runs on the SIMT kernels
    (bf16 operands read as fp32, fp32 sums, RNE outputs) and matches the
    oracle like the tensor-core backward does."""
    N = 384
    q, k, v, do = _inputs(torch.bfloat16, 2, 4, 2, N, d, 5 + d)
    o_ref, l_ref = oatt.attention_forward(np64(q), np64(k), np64(v), causal=True)
    g_ref = oatt.attention_backward(np64(q), np64(k), np64(v), np64(do), causal=True)
    perm = lambda x: rm.layout_permute(x.cuda(), layout, P)
    unperm = lambda x: rm.layout_permute(x, layout, P, inverse=True)
    qr, kr, vr, dor = perm(q), perm(k), perm(v), perm(do)
    o, l = rm.ring_attn_fwd(qr, kr, vr, P=P, layout=layout, causal=True)
    assert_max_abs(np64(unperm(o)), o_ref, BF16_O_TOL, "O")
    grads = rm.ring_attn_bwd(qr, kr, vr, o, l, dor, P=P, layout=layout, causal=True)
    for name, g, ref in zip(("dq", "dk", "dv"), grads, g_ref):
        assert g.dtype == torch.bfloat16
        assert_grad_close(np64(unperm(g)), ref, what=name)
    # global token order in the backward needs the tensor-core path (d = 128)
    if layout != "contiguous":
        with pytest.raises(rm.RmError) as e:
            rm.ring_attn_bwd(q.cuda(), k.cuda(), v.cuda(), o, l, do.cuda(), P=P, layout=layout,
                             causal=True, order="global")
        assert e.value.status == rm.RM_ERR_UNSUPPORTED


def test_bf16_block_backward_head_dim_64(rm):
    """The block API at d = 64 accumulates one shard pair's gradients in fp32."""
    N, P, d = 256, 2, 64
    q, k, v, do = _inputs(torch.bfloat16, 1, 4, 2, N, d, 17)
    L = N // P
    f64 = lambda t: np64(t)
    qs, ks, vs, dos = q[:, L:], k[:, :L], v[:, :L], do[:, L:]
    o_ref, l_ref = oatt.attention_forward(f64(q), f64(k), f64(v), causal=True)
    delta = oatt.delta_from_output(f64(do), o_ref)
    ref = oatt.attention_backward_block(f64(qs), f64(ks), f64(vs), f64(dos), l_ref[:, :, L:],
                                        delta[:, :, L:], causal=True,
                                        q_pos=np.arange(L, N), k_pos=np.arange(0, L))
    dq = torch.zeros(1, L, 4, d, device="cuda")
    dk = torch.zeros(1, L, 2, d, device="cuda")
    dv = torch.zeros(1, L, 2, d, device="cuda")
    lse = torch.from_numpy(np.ascontiguousarray(l_ref[:, :, L:])).float().cuda()
    dlt = torch.from_numpy(np.ascontiguousarray(delta[:, :, L:])).float().cuda()
    rm.attn_block_bwd(qs.cuda().contiguous(), ks.cuda().contiguous(), vs.cuda().contiguous(),
                      dos.cuda().contiguous(), lse, dlt, dq, dk, dv, N=N, P=P,
                      layout="contiguous", causal=True, q_rank=1, kv_rank=0)
    for name, g, r in zip(("dq", "dk", "dv"), (dq, dk, dv), ref):
        assert_grad_close(np64(g), r, what=name)


def _global_ok(case):
    dtype, B, Hq, Hkv, N, d, P, layout, causal = case
    return layout != "zigzag" or (N // (2 * P)) % 128 == 0


GLOBAL_CASES = [c for c in CASES if c[0] == torch.bfloat16 and _global_ok(c)] + [
    (torch.bfloat16, 1, 4, 2, 1024, 64, 2, "zigzag", True),
    (torch.bfloat16, 1, 4, 2, 1024, 32, 8, "striped", True),
]


def _lse_unpermute(rm, lse, layout, P):
    B, H, N = lse.shape
    flat = lse.reshape(B * H, N, 1, 1).contiguous()
    return rm.layout_permute(flat, layout, P, inverse=True).reshape(B, H, N)


@pytest.mark.parametrize("case", GLOBAL_CASES, ids=lambda c: f"B{c[1]}H{c[2]}/{c[3]}-N{c[4]}-d{c[5]}-P{c[6]}-{c[7]}-{'c' if c[8] else 'nc'}")
def test_ring_global_order_matches_rank_major(rm, case):
    """Global-order operands (the kernels fetch each rank's tiles through the
    layout) give bit-for-bit the results of permute -> rank-major ring ->
    un-permute, forward and (d = 128) backward."""
    dtype, B, Hq, Hkv, N, d, P, layout, causal = case
    q, k, v, do = (t.cuda() for t in _inputs(dtype, B, Hq, Hkv, N, d, 330 + N))
    perm = lambda x: rm.layout_permute(x, layout, P)
    unperm = lambda x: rm.layout_permute(x, layout, P, inverse=True)
    qr, kr, vr, dor = perm(q), perm(k), perm(v), perm(do)
    o_r, l_r = rm.ring_attn_fwd(qr, kr, vr, P=P, layout=layout, causal=causal)
    o_g, l_g = rm.ring_attn_fwd(q, k, v, P=P, layout=layout, causal=causal, order="global")
    assert torch.equal(o_g, unperm(o_r))
    assert torch.equal(l_g, _lse_unpermute(rm, l_r, layout, P))
    if d != 128:
        return
    grads_r = rm.ring_attn_bwd(qr, kr, vr, o_r, l_r, dor, P=P, layout=layout, causal=causal)
    grads_g = rm.ring_attn_bwd(q, k, v, o_g, l_g, do, P=P, layout=layout, causal=causal,
                               order="global")
    for name, gr, gg in zip(("dq", "dk", "dv"), grads_r, grads_g):
        assert torch.equal(gg, unperm(gr)), name


def test_ring_global_order_against_oracle(rm):
    """One global-order case straight against the oracle (no permutes at all)."""
    case = (torch.bfloat16, 1, 4, 2, 2048, 128, 4, "zigzag", True)
    dtype, B, Hq, Hkv, N, d, P, layout, causal = case
    q, k, v, do = _inputs(dtype, B, Hq, Hkv, N, d, 777)
    o_ref, l_ref = oatt.attention_forward(np64(q), np64(k), np64(v), causal=True)
    g_ref = oatt.attention_backward(np64(q), np64(k), np64(v), np64(do), causal=True)
    qg, kg, vg, dog = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    o, l = rm.ring_attn_fwd(qg, kg, vg, P=P, layout=layout, causal=True, order="global")
    assert_max_abs(np64(o), o_ref, BF16_O_TOL, "O")
    assert_max_abs(np64(l), l_ref, BF16_LSE_TOL, "LSE")
    grads = rm.ring_attn_bwd(qg, kg, vg, o, l, dog, P=P, layout=layout, causal=True, order="global")
    for name, g, ref in zip(("dq", "dk", "dv"), grads, g_ref):
        assert_grad_close(np64(g), ref, what=name)
