"""Full-size parity of the ring forward + backward at the three bf16 causal
workloads (16k zigzag P=2, 128k striped P=8, 256k zigzag P=8): the
rank-major ring (after a layout permute) is checked against the oracle, and
the launch configuration bench.py times (fused ring forward and ring
backward on global-order operands, K and V as views of one fused buffer)
must reproduce its results bit for bit.

The oracle cannot materialise these problems, so it checks what it can
compute exactly one by one:
- O, LSE and dQ of sampled query rows (each needs only its own score row);
- dK and dV of the last keys of the sequence: every query that sees them lies
  in the tail window, whose rows the oracle computes in full;
- at every key, the invariants sum_u dK_u = 0 and sum_u dV_u = sum_t dO_t
  (per batch and KV head), which hold at any size.
"""

import numpy as np
import pytest
import torch

from oracle import attention as oatt
from sequence_attention_rm_b200 import synthetic
from tests._helpers import BF16_LSE_TOL, BF16_O_TOL, assert_grad_close, assert_max_abs, gpu

pytestmark = gpu

TAIL = 256


@pytest.fixture(scope="module")
def rm():
    from sequence_attention_rm_b200 import rm as mod
    return mod


def _sample_rows(w, n_random, seed):
    """Global positions: sequence ends, every zigzag chunk / rank edge, random."""
    N, P = w.N, w.P
    edges = set([0, 1, N - 1, N - 2])
    for c in range(2 * P + 1):
        for x in (c * N // (2 * P) - 1, c * N // (2 * P)):
            if 0 <= x < N:
                edges.add(x)
    rng = np.random.default_rng(seed)
    edges.update(rng.integers(0, N, n_random).tolist())
    return np.array(sorted(edges), dtype=np.int64)


def _f64(t):
    return t.to(torch.float64).numpy()


@pytest.mark.parametrize("w", [synthetic.LLAMA_ZIGZAG, synthetic.STRIPED_128K,
                               synthetic.LONG_ZIGZAG_256K], ids=lambda w: w.name)
def test_full_size_ring_fwd_bwd(rm, w):
    q, k, v, do = synthetic.attention_inputs(w)
    dev = torch.device("cuda")
    perm = lambda x: rm.layout_permute(x.to(dev), w.layout, w.P)
    qr, kr, vr, dor = perm(q), perm(k), perm(v), perm(do)
    o, lse = rm.ring_attn_fwd(qr, kr, vr, P=w.P, layout=w.layout, causal=True)
    dq, dk, dv = rm.ring_attn_bwd(qr, kr, vr, o, lse, dor, P=w.P, layout=w.layout, causal=True)
    back = lambda x: rm.layout_permute(x, w.layout, w.P, inverse=True).cpu()
    o_g, dq_g, dk_g, dv_g = back(o), back(dq), back(dk), back(dv)
    lse_g = rm.layout_permute(lse.view(w.Hq, w.N, 1, 1), w.layout, w.P, inverse=True).view(
        w.B, w.Hq, w.N).cpu()
    del qr, kr, vr, dor, o, lse, dq, dk, dv
    torch.cuda.empty_cache()
    # the launch configuration bench.py times: the same ring on global-order
    # operands (no permute pass) must give the same bits
    qd, kd, vd, dod = q.to(dev), k.to(dev), v.to(dev), do.to(dev)
    og, lg = rm.ring_attn_fwd(qd, kd, vd, P=w.P, layout=w.layout, causal=True, order="global")
    grads = rm.ring_attn_bwd(qd, kd, vd, og, lg, dod, P=w.P, layout=w.layout, causal=True,
                             order="global")
    assert torch.equal(og.cpu(), o_g) and torch.equal(lg.cpu(), lse_g), "global-order forward"
    for name, a, ref in zip(("dq", "dk", "dv"), grads, (dq_g, dk_g, dv_g)):
        assert torch.equal(a.cpu(), ref), f"global-order {name}"
    del kd, vd, og, lg, grads
    torch.cuda.empty_cache()
    # ... and with K and V as head views of one fused [B, N, 2 Hkv, d] buffer
    # (K heads first), the operand form bench.py times
    kv = torch.cat([k, v], dim=2).to(dev)
    kf, vf = kv[:, :, :w.Hkv], kv[:, :, w.Hkv:]
    og, lg = rm.ring_attn_fwd(qd, kf, vf, P=w.P, layout=w.layout, causal=True, order="global")
    grads = rm.ring_attn_bwd(qd, kf, vf, og, lg, dod, P=w.P, layout=w.layout, causal=True,
                             order="global")
    assert torch.equal(og.cpu(), o_g) and torch.equal(lg.cpu(), lse_g), "fused K|V forward"
    for name, a, ref in zip(("dq", "dk", "dv"), grads, (dq_g, dk_g, dv_g)):
        assert torch.equal(a.cpu(), ref), f"fused K|V {name}"
    del qd, kv, kf, vf, dod, og, lg, grads
    torch.cuda.empty_cache()
    assert rm.get_device_status() == rm.RM_OK

    rows = _sample_rows(w, 48, w.wid)
    tail = np.arange(w.N - TAIL, w.N, dtype=np.int64)
    group = w.Hq // w.Hkv
    for g in range(w.Hkv):
        kk, vv = _f64(k[:, :, g:g + 1]), _f64(v[:, :, g:g + 1])
        for h in range(g * group, (g + 1) * group):
            qh, doh = q[:, :, h:h + 1], do[:, :, h:h + 1]
            # sampled rows: O, LSE, dQ
            qs, dos = _f64(qh[:, rows]), _f64(doh[:, rows])
            o_ref, l_ref = oatt.attention_forward(qs, kk, vv, causal=True, q_pos=rows)
            assert_max_abs(o_g[:, rows, h:h + 1].double().numpy(), o_ref, BF16_O_TOL, f"O h{h}")
            assert_max_abs(lse_g[:, h:h + 1, rows].double().numpy(), l_ref, BF16_LSE_TOL, f"LSE h{h}")
            delta = oatt.delta_from_output(dos, o_ref)
            dq_ref, _, _ = oatt.attention_backward_block(qs, kk, vv, dos, l_ref, delta, causal=True,
                                                         q_pos=rows)
            assert_grad_close(dq_g[:, rows, h:h + 1].double().numpy(), dq_ref, what=f"dQ h{h}")
        # tail keys: every query that sees them is in the tail window
        dk_ref = np.zeros((1, TAIL, 1, w.d))
        dv_ref = np.zeros((1, TAIL, 1, w.d))
        for h in range(g * group, (g + 1) * group):
            qt, dot = _f64(q[:, tail, h:h + 1]), _f64(do[:, tail, h:h + 1])
            o_t, l_t = oatt.attention_forward(qt, kk, vv, causal=True, q_pos=tail)
            delta = oatt.delta_from_output(dot, o_t)
            _, gk, gv = oatt.attention_backward_block(qt, kk[:, tail], vv[:, tail], dot, l_t, delta,
                                                      causal=True, q_pos=tail, k_pos=tail)
            dk_ref += gk
            dv_ref += gv
        assert_grad_close(dk_g[:, tail, g:g + 1].double().numpy(), dk_ref, what=f"dK tail g{g}")
        assert_grad_close(dv_g[:, tail, g:g + 1].double().numpy(), dv_ref, what=f"dV tail g{g}")
        # invariants over every key, per head-dim column: the exact sums are
        # 0 and sum_t dO_t; each stored element is off by at most ~1e-2 of
        # its own magnitude (bf16 rounding of P / dS / the output), so the
        # sums may be off by 1e-2 of the L1 norm of the column
        dkc, dvc = dk_g[:, :, g].double(), dv_g[:, :, g].double()
        sdo = do[:, :, g * group:(g + 1) * group].double().sum(dim=(1, 2))
        assert (dkc.sum(dim=1).abs() <= 1e-2 * dkc.abs().sum(dim=1) + 1e-6).all(), "sum_u dK_u = 0"
        assert ((dvc.sum(dim=1) - sdo).abs() <= 1e-2 * dvc.abs().sum(dim=1) + 1e-6).all(), \
            "sum_u dV_u = sum_t dO_t"
