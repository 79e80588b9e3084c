"""The tabular multi-axis workload: a (batch, rows, features, embed) bf16
tensor with 4 heads of d=24.  Row-axis attention runs as a non-causal ring
over P=8 contiguous shards on strided head views (no copy; d zero-padded to 32
on chip); feature-axis attention (5 tokens) runs on the short-sequence kernel.
Compared with the oracle's multi-axis routing."""

import numpy as np
import pytest
import torch

from oracle import attention as oatt
from oracle import multiaxis as omulti
from sequence_attention_rm_b200 import synthetic
from tests._helpers import BF16_LSE_TOL, BF16_O_TOL, assert_max_abs, gpu, np64

pytestmark = gpu


@pytest.fixture(scope="module")
def rm():
    from sequence_attention_rm_b200 import rm as mod
    return mod


def _row_axis(rm, q, k, v, w, mode):
    R, F, E, H = w.rows, w.features, w.embed, w.heads
    view = lambda x: x.view(w.batch, R, F * H, E // H)   # head index f*H + h; strided, no copy
    o, lse = rm.ring_attn_fwd(view(q), view(k), view(v), P=w.P, layout="contiguous",
                              causal=False, mode=mode)
    return o.view(w.batch, R, F, E), lse


def _feature_axis(rm, q, k, v, w):
    R, F, E, H = w.rows, w.features, w.embed, w.heads
    view = lambda x: x.view(w.batch * R, F, H, E // H)
    o, lse = rm.attn_block_fwd(view(q), view(k), view(v), N=F, P=1, layout="contiguous",
                               causal=False, q_rank=0, kv_rank=0)
    return o.view(w.batch, R, F, E), lse


@pytest.mark.parametrize("rows", [1000, 2048 + 8 * 37])
@pytest.mark.parametrize("mode", ["fused", "stepwise"])
def test_tabular_small(rm, rows, mode):
    w = synthetic.TABULAR.scaled(rows)
    q, k, v = (t.cuda() for t in synthetic.tabular_inputs(w))
    o_ref, l_ref = omulti.row_axis_attention(np64(q), np64(k), np64(v), w.heads)
    o, l = _row_axis(rm, q, k, v, w, mode)
    assert_max_abs(np64(o), o_ref, BF16_O_TOL, "row-axis O")
    assert_max_abs(np64(l), l_ref, BF16_LSE_TOL, "row-axis LSE")
    fo_ref, fl_ref = omulti.feature_axis_attention(np64(q), np64(k), np64(v), w.heads)
    fo, fl = _feature_axis(rm, q, k, v, w)
    assert_max_abs(np64(fo), fo_ref, BF16_O_TOL, "feature-axis O")
    assert_max_abs(np64(fl), fl_ref, BF16_LSE_TOL, "feature-axis LSE")


def test_tabular_same_tensor_qkv(rm):
    w = synthetic.TABULAR.scaled(1200)
    x = synthetic.tabular_inputs(w)[0].cuda()
    o_ref, l_ref = omulti.row_axis_attention(np64(x), np64(x), np64(x), w.heads)
    o, l = _row_axis(rm, x, x, x, w, "fused")
    assert_max_abs(np64(o), o_ref, BF16_O_TOL, "row-axis O (q=k=v)")
    assert_max_abs(np64(l), l_ref, BF16_LSE_TOL, "row-axis LSE (q=k=v)")


def test_tabular_full_size_sampled(rm):
    w = synthetic.TABULAR
    qc, kc, vc = synthetic.tabular_inputs(w)
    q, k, v = qc.cuda(), kc.cuda(), vc.cuda()
    o, l = _row_axis(rm, q, k, v, w, "fused")
    fo, fl = _feature_axis(rm, q, k, v, w)
    o, l, fo, fl = o.cpu(), l.cpu(), fo.cpu(), fl.cpu()
    assert rm.get_device_status() == rm.RM_OK
    R, F, E, H = w.rows, w.features, w.embed, w.heads
    dh = E // H
    rng = np.random.default_rng(4)
    rows = np.unique(np.concatenate([[0, R - 1], np.arange(8) * (R // 8),
                                     np.arange(1, 9) * (R // 8) - 1, rng.integers(0, R, 24)]))
    # row axis: every (feature, head) sequence, sampled query rows, all 150000 keys
    for f in range(F):
        for h in range(H):
            cs = slice(h * dh, (h + 1) * dh)
            qq = np64(qc[:, rows, f, cs])[:, :, None]
            kk = np64(kc[:, :, f, cs])[:, :, None]
            vv = np64(vc[:, :, f, cs])[:, :, None]
            o_ref, l_ref = oatt.attention_forward(qq, kk, vv, q_pos=rows)
            assert_max_abs(np64(o[:, rows, f, cs]), o_ref[:, :, 0], BF16_O_TOL, f"row O f{f} h{h}")
            assert_max_abs(np64(l[:, f * H + h, rows]), l_ref[:, 0], BF16_LSE_TOL, f"row LSE f{f} h{h}")
    # feature axis: sampled rows, in full
    fr = np.sort(rng.choice(R, 3000, replace=False))
    sub = lambda t: np64(t[:, fr])
    fo_ref, fl_ref = omulti.feature_axis_attention(sub(qc), sub(kc), sub(vc), H)
    assert_max_abs(np64(fo[:, fr]), fo_ref, BF16_O_TOL, "feature O")
    assert_max_abs(np64(fl[fr]), fl_ref, BF16_LSE_TOL, "feature LSE")
