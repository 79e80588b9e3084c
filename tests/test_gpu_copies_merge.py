"""GPU parity of the bandwidth-bound kernels against the oracle: layout
permute and Ulysses repack (bit-exact), LSE merge and the backward
preprocess (fp32 tolerance), and the bounded-wait status machinery."""

import numpy as np
import pytest
import torch

from oracle import attention as oatt
from oracle import layouts as olay
from oracle import merge as omerge
from oracle import repack as orepack
from sequence_attention_rm_b200 import synthetic
from tests._helpers import BF16_O_TOL, F32_TOL, assert_f32_close, assert_max_abs, gpu, np64

pytestmark = gpu


@pytest.fixture(scope="module")
def rm():
    from sequence_attention_rm_b200 import rm as mod
    return mod


def _bits(t: torch.Tensor) -> np.ndarray:
    t = t.detach().cpu().contiguous()
    return t.view(torch.int16).numpy() if t.dtype == torch.bfloat16 else t.view(torch.int32).numpy()


@pytest.mark.parametrize("layout", ["contiguous", "zigzag", "striped"])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("B,N,H,d,P", [(1, 64, 2, 8, 2), (2, 1000, 3, 24, 4), (1, 4096, 16, 128, 8),
                                       (1, 48, 1, 3, 2), (1, 96, 5, 1, 4)])
def test_layout_permute_bit_exact(rm, layout, dtype, B, N, H, d, P):
    if layout == "zigzag" and N % (2 * P):
        pytest.skip("zigzag needs 2P | N")
    x = synthetic.tensor(11 + N, (B, N, H, d), dtype)
    ref = olay.permute(_bits(x), layout, P)
    y = rm.layout_permute(x.cuda(), layout, P)
    assert np.array_equal(_bits(y), ref)
    back = rm.layout_permute(y, layout, P, inverse=True)
    assert np.array_equal(_bits(back), _bits(x))


def test_layout_permute_empty(rm):
    x = torch.empty((1, 0, 4, 8), dtype=torch.bfloat16, device="cuda")
    assert rm.layout_permute(x, "zigzag", 2).shape == x.shape


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("P,L,H,d", [(1, 5, 2, 8), (2, 7, 4, 8), (8, 33, 16, 128), (4, 3, 8, 3),
                                     (8, 2, 16, 24)])
def test_seq_head_repack_bit_exact(rm, dtype, P, L, H, d):
    x = synthetic.tensor(97 + L, (P, L, H, d), dtype)
    ref = orepack.seq_to_head(_bits(x), P)
    y = rm.seq_head_repack(x.cuda(), P)
    assert np.array_equal(_bits(y), ref)
    back = rm.seq_head_repack(y, P, head_to_seq=True)
    assert np.array_equal(_bits(back), _bits(x))
    assert np.array_equal(orepack.head_to_seq(ref, P), _bits(x))


@pytest.mark.parametrize("L", [2048, 32768], ids=["8x2048", "8x32768-full"])
def test_repack_workload_shapes(rm, L):
    """The 256k zigzag workload's repack at its full size (L = 32768 tokens per
    rank; 1 GiB per tensor) and at 1/16 of it: Q [8 x L, 16, 128], the fused
    K|V (8 K heads then 8 V heads) of the same shape, and K alone
    [8 x L, 8, 128], sequence-sharded -> head-sharded and back, bit for bit
    against the oracle's index loops."""
    for seed, H in ((5000, 16), (5001, 16), (5002, 8)):
        x = synthetic.tensor(seed + L, (8, L, H, 128), torch.bfloat16)
        xb = _bits(x)
        xd = x.cuda()
        y = rm.seq_head_repack(xd, 8)
        assert y.shape == (8, 8 * L, H // 8, 128)
        ref = orepack.seq_to_head(xb, 8)
        assert np.array_equal(_bits(y), ref)
        # head -> seq on the oracle's head-sharded tensor (not on the kernel's)
        back = rm.seq_head_repack(torch.from_numpy(ref).view(torch.bfloat16).cuda(), 8,
                                  head_to_seq=True)
        assert np.array_equal(_bits(back), orepack.head_to_seq(ref, 8))
        assert np.array_equal(_bits(back), xb)
        del xd, y, back
        torch.cuda.empty_cache()


@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("n,B,H,Nq,d", [(1, 1, 2, 5, 8), (2, 1, 3, 77, 64), (4, 2, 4, 130, 128),
                                        (8, 1, 16, 300, 128), (3, 1, 2, 33, 24), (16, 1, 1, 9, 4),
                                        (2, 2, 3, 77, 128), (2, 1, 2, 31, 128)])
def test_lse_merge(rm, out_dtype, n, B, H, Nq, d):
    o_parts = [synthetic.tensor(300 + i, (B, Nq, H, d)) for i in range(n)]
    lse_parts = [synthetic.tensor(400 + i, (B, H, Nq), scale=3.0) for i in range(n)]
    # empty partials (no visible key): lse = -inf, O = 0
    if n > 1:
        lse_parts[1][..., ::3] = -np.inf
        o_parts[1][:, ::3] = 0.0
    lse_parts[0][..., 1] = -np.inf
    for p in lse_parts[1:]:
        p[..., 1] = -np.inf  # a row where every partial is empty
    for p in o_parts:
        p[:, 1] = 0.0
    ref_o, ref_l = omerge.lse_merge([np64(o) for o in o_parts], [np64(l) for l in lse_parts])
    o, l = rm.lse_merge([o.cuda() for o in o_parts], [l.cuda() for l in lse_parts], out_dtype)
    # bf16 output: O values reach ~8 here, where one bf16 half-ulp is 2^-9 * 8
    tol = F32_TOL if out_dtype == torch.float32 else BF16_O_TOL
    assert_max_abs(np64(o), ref_o, tol, "merged O")
    assert_max_abs(np64(l), ref_l, 1e-5, "merged LSE")
    assert np.all(np.isneginf(np64(l)[..., 1]))


@pytest.mark.parametrize("n,Nq,H,d", [(3, 50, 2, 32), (2, 1001, 3, 128), (2, 517, 2, 64)])
def test_lse_merge_in_place(rm, n, Nq, H, d):
    # several rows per warp pass for two partials: row counts that leave a pass partly empty
    o_parts = [synthetic.tensor(700 + i, (1, Nq, H, d)).cuda() for i in range(n)]
    lse_parts = [synthetic.tensor(710 + i, (1, H, Nq)).cuda() for i in range(n)]
    ref_o, ref_l = omerge.lse_merge([np64(o) for o in o_parts], [np64(l) for l in lse_parts])
    rm.lse_merge(o_parts, lse_parts, torch.float32, out=o_parts[0], lse_out=lse_parts[0])
    assert_max_abs(np64(o_parts[0]), ref_o, F32_TOL)
    assert_max_abs(np64(lse_parts[0]), ref_l, 1e-5)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("B,N,H,d", [(1, 7, 3, 128), (2, 130, 16, 128), (1, 33, 20, 24), (1, 5, 2, 4),
                                     (3, 65, 8, 64), (1, 40, 5, 32), (1, 9, 3, 12)])
def test_bwd_preprocess(rm, dtype, B, N, H, d):
    o = synthetic.tensor(800, (B, N, H, d), dtype)
    do = synthetic.tensor(801, (B, N, H, d), dtype)
    ref = oatt.delta_from_output(np64(do), np64(o))
    got = rm.attn_bwd_preprocess(o.cuda(), do.cuda())
    assert_f32_close(np64(got), ref, "delta")


def test_bounded_wait_reports_timeout_and_context_survives(rm):
    assert rm.get_device_status() == rm.RM_OK
    rm.debug_expire_wait(1000)
    assert rm.get_device_status() == rm.RM_ERR_TIMEOUT
    assert rm.get_device_status() == rm.RM_OK  # the status word was cleared
    x = torch.arange(16, device="cuda", dtype=torch.float32).reshape(1, 4, 1, 4)
    y = rm.layout_permute(x, "striped", 2)      # the context still works
    assert torch.equal(rm.layout_permute(y, "striped", 2, inverse=True), x)


def test_launch_profiler_records_each_launch(rm):
    x = synthetic.tensor(31, (1, 256, 4, 64), torch.bfloat16).cuda()
    rm.profile_enable(True)
    y = rm.layout_permute(x, "zigzag", 2)
    rm.seq_head_repack(y.view(2, 128, 4, 64), 2)
    recs = rm.profile_records()
    rm.profile_enable(False)
    assert [n for n, _ in recs] == ["layout_permute", "seq_head_repack"]
    assert all(ms > 0 for _, ms in recs)
    rm.layout_permute(x, "zigzag", 2)
    assert rm.profile_records() == []  # disabled: nothing recorded


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_lse_merge_mixed_strides(rm, out_dtype, d):
    """Partials whose strides differ (a head view of a wider tensor, a dense
    tensor) and an output view with its own strides."""
    B, Nq, H = 2, 301, 3
    wide = synthetic.tensor(920, (B, Nq, H + 2, d)).cuda()
    o_parts = [wide[:, :, 1:1 + H], synthetic.tensor(921, (B, Nq, H, d)).cuda()]
    lse_parts = [synthetic.tensor(930 + i, (B, H, Nq), scale=3.0).cuda() for i in range(2)]
    ref_o, ref_l = omerge.lse_merge([np64(o) for o in o_parts], [np64(l) for l in lse_parts])
    out_wide = torch.zeros(B, Nq, H + 1, d, dtype=out_dtype, device="cuda")
    out = out_wide[:, :, :H]
    o, l = rm.lse_merge(o_parts, lse_parts, out_dtype, out=out)
    tol = F32_TOL if out_dtype == torch.float32 else BF16_O_TOL
    assert_max_abs(np64(out), ref_o, tol, "merged O")
    assert_max_abs(np64(l), ref_l, 1e-5, "merged LSE")
    assert not out_wide[:, :, H].any()  # the column outside the view is untouched


@pytest.mark.parametrize("offset", [8, 4])
def test_bwd_preprocess_strided_views(rm, offset):
    """Head views inside wider rows: 16-byte aligned rows (offset 8 elements)
    take the 16-byte-lane kernel, 8-byte aligned rows (offset 4) the 8-byte one."""
    B, N, H, d = 2, 77, 6, 64
    wide_o = synthetic.tensor(810, (B, N, H, d + 16), torch.bfloat16).cuda()
    wide_do = synthetic.tensor(811, (B, N, H, d + 16), torch.bfloat16).cuda()
    o, do = wide_o[..., offset:offset + d], wide_do[..., offset:offset + d]
    ref = oatt.delta_from_output(np64(do), np64(o))
    got = rm.attn_bwd_preprocess(o, do)
    assert_f32_close(np64(got), ref, "delta")
