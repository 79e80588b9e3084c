"""The C-ABI library loads, exports every entry point its header declares, and
rejects bad arguments on the host before any launch (no GPU needed)."""

import ctypes
import os
import re

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "rm_attn.h")


def _declared():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^(?:rm_status|const char\*)\s+(rm_\w+)\(", text, re.M)))


@pytest.fixture(scope="module")
def rm():
    from sequence_attention_rm_b200 import rm as mod
    return mod


def test_header_declares_the_boundary():
    names = _declared()
    for must in ("rm_attn_block_fwd", "rm_attn_block_bwd", "rm_lse_merge", "rm_ring_attn_fwd",
                 "rm_ring_attn_bwd", "rm_seq_head_repack", "rm_layout_permute",
                 "rm_ring_workspace_size", "rm_get_device_status"):
        assert must in names


def test_library_exports_every_declared_symbol(rm):
    lib = rm.raw()
    for name in _declared():
        assert hasattr(lib, name), name
    assert set(_declared()) <= set(rm.EXPORTED) | {"rm_status_string", "rm_last_error"}


def test_status_strings(rm):
    lib = rm.raw()
    assert lib.rm_status_string(0) == b"RM_OK"
    assert lib.rm_status_string(5) == b"RM_ERR_TIMEOUT"


def _desc(rm, **kw):
    base = dict(dtype=rm.RM_BF16, B=1, Hq=16, Hkv=8, d=128, N=16384, P=2, layout=1, causal=1,
                scale=0.0, mode=0)
    base.update(kw)
    return rm.RmAttnDesc(**base)


@pytest.mark.parametrize("bad,status", [
    (dict(d=96), 2),            # unsupported bf16 head dim
    (dict(Hq=12, Hkv=8), 1),    # Hq % Hkv != 0
    (dict(N=1000, P=3), 1),     # N % P != 0
    (dict(N=4100, P=4), 1),     # zigzag needs N % 2P == 0
    (dict(layout=7), 1),        # bad layout
    (dict(P=0), 1),
    (dict(dtype=9), 1),
    (dict(dtype=0, d=130), 2),  # fp32 d > 128
    (dict(mode=3), 1),
    (dict(order=5), 1),                      # bad token order
    (dict(order=1, N=2000, P=2), 2),         # global zigzag: chunk of 500 tokens
    (dict(order=1, dtype=0), 2),             # global order needs bf16
    (dict(order=1, mode=1), 2),              # global order needs the fused forward
    (dict(N=1 << 31), 1),                    # positions are 32-bit on the device
    # segments (the pointers are never read by the validation)
    (dict(cu_seqlens=16, num_segments=2, seq_lens=16), 1),  # exclusive
    (dict(cu_seqlens=16, num_segments=2, B=2), 1),          # packing needs B == 1
    (dict(cu_seqlens=16, num_segments=0), 1),
])
def test_desc_validation(rm, bad, status):
    n = ctypes.c_size_t(0)
    d = _desc(rm, **bad)
    assert rm.raw().rm_ring_workspace_size(ctypes.byref(d), 0, ctypes.byref(n)) == status
    assert rm.raw().rm_last_error()


@pytest.mark.parametrize("kw", [dict(seq_lens=16, dtype=0), dict(cu_seqlens=16, num_segments=3, dtype=0),
                                dict(seq_lens=16), dict(cu_seqlens=16, num_segments=3)])
def test_desc_accepts_segments(rm, kw):
    """Packed and right-padded batches in bf16 (tensor-core kernels) and fp32
    (SIMT kernels)."""
    n = ctypes.c_size_t(0)
    d = _desc(rm, **kw)
    for backward in (0, 1):
        assert rm.raw().rm_ring_workspace_size(ctypes.byref(d), backward, ctypes.byref(n)) == 0


def test_global_order_accepted(rm):
    n = ctypes.c_size_t(0)
    lib = rm.raw()
    for kw in (dict(order=1), dict(order=1, layout=2, P=8), dict(order=1, layout=0, dtype=0, mode=1),
               dict(order=1, P=1, dtype=0, mode=1, N=1000)):
        d = _desc(rm, **kw)
        assert lib.rm_ring_workspace_size(ctypes.byref(d), 0, ctypes.byref(n)) == 0, kw
        assert lib.rm_ring_workspace_size(ctypes.byref(d), 1, ctypes.byref(n)) == 0, kw


def test_workspace_sizes(rm):
    n = ctypes.c_size_t(0)
    lib = rm.raw()
    d = _desc(rm)
    assert lib.rm_ring_workspace_size(ctypes.byref(d), 0, ctypes.byref(n)) == 0
    assert n.value == 0  # fused forward needs no workspace
    assert lib.rm_ring_workspace_size(ctypes.byref(d), 1, ctypes.byref(n)) == 0
    # delta [B, Hq, N]: the backward kernels write dQ / dK / dV directly
    assert n.value == 16 * 16384 * 4
    d = _desc(rm, mode=1)
    assert lib.rm_ring_workspace_size(ctypes.byref(d), 0, ctypes.byref(n)) == 0
    assert n.value == 2 * 16 * 16384 * 128 * 4 + 2 * 16 * 16384 * 4


def test_entry_points_reject_bad_arguments_before_launch(rm):
    lib = rm.raw()
    nul = ctypes.c_void_p(0)
    # layout permute: bad layout, N % P, overlapping buffers, NULL pointers
    assert lib.rm_layout_permute(1, 1, 64, 2, 8, 9, 2, 0, nul, nul, nul) == 1
    assert lib.rm_layout_permute(1, 1, 63, 2, 8, 0, 2, 0, nul, nul, nul) == 1
    assert lib.rm_layout_permute(1, 1, 64, 2, 8, 0, 2, 0, nul, nul, nul) == 1
    buf = ctypes.create_string_buffer(4096)
    p = ctypes.cast(buf, ctypes.c_void_p)
    assert lib.rm_layout_permute(1, 1, 64, 2, 8, 0, 2, 0, p, p, nul) == 1  # overlap
    assert lib.rm_layout_permute(1, 0, 64, 2, 8, 0, 2, 0, nul, nul, nul) == 0  # empty: no-op
    # repack: head count must be a multiple of P (the Ulysses cap)
    assert lib.rm_seq_head_repack(1, 4, 8, 6, 8, 0, nul, nul, nul) == 1
    assert lib.rm_seq_head_repack(1, 4, 0, 8, 8, 0, nul, nul, nul) == 0
    # merge: too many parts, bad head dim
    T = rm.RmTensor
    parts = (T * 1)(T(0, 0, 0, 0))
    lses = (ctypes.c_void_p * 1)(0)
    assert lib.rm_lse_merge(1, 1, 2, 8, 64, 17, parts, lses, T(0, 0, 0, 0), nul, nul) == 1
    assert lib.rm_lse_merge(1, 1, 2, 8, 66, 1, parts, lses, T(0, 0, 0, 0), nul, nul) == 1
    # ring forward: misaligned pointer / strides
    d = _desc(rm, N=256, P=2)
    bad_ptr = T(p.value + 8, 256 * 16 * 128, 16 * 128, 128)
    ok = T(p.value, 256 * 16 * 128, 16 * 128, 128)
    assert lib.rm_ring_attn_fwd(ctypes.byref(d), bad_ptr, ok, ok, ok, p, nul, 0, nul) == 1
    bad_stride = T(p.value, 256 * 16 * 128, 16 * 128 + 3, 128)
    assert lib.rm_ring_attn_fwd(ctypes.byref(d), ok, bad_stride, ok, ok, p, nul, 0, nul) == 1
    # ring backward without a workspace
    kv = T(p.value, 256 * 8 * 128, 8 * 128, 128)
    assert lib.rm_ring_attn_bwd(ctypes.byref(d), ok, kv, kv, ok, p, ok, ok, kv, kv, nul, 0,
                                nul) == 3
    # block forward: rank out of range
    assert lib.rm_attn_block_fwd(ctypes.byref(d), 2, 0, ok, kv, kv, ok, 0, p, nul) == 1
    # fp32 -> out dtype conversion: dtype, sizes, NULL, alignment; empty is a no-op
    src = T(p.value, 256 * 16 * 128, 16 * 128, 128)
    dst = T(p.value + 2048, 256 * 16 * 128, 16 * 128, 128)
    assert lib.rm_convert_f32(2, 1, 256, 16, 128, src, dst, nul) == 1  # no dtype 2
    assert lib.rm_convert_f32(1, 1, 256, 16, 126, src, dst, nul) == 1  # d % 4
    assert lib.rm_convert_f32(1, 1, 256, 0, 128, src, dst, nul) == 1  # H < 1
    assert lib.rm_convert_f32(1, 1, 256, 16, 128, T(0, 0, 0, 0), dst, nul) == 1  # NULL
    assert lib.rm_convert_f32(1, 1, 256, 16, 128, T(p.value + 4, 256 * 16 * 128, 16 * 128, 128),
                              dst, nul) == 1  # fp32 input off a 16-byte boundary
    assert lib.rm_convert_f32(1, 1, 256, 16, 128, src, T(p.value + 2, 256 * 16 * 128, 16 * 128,
                                                         128), nul) == 1  # bf16 output off 8 bytes
    assert lib.rm_convert_f32(1, 0, 256, 16, 128, T(0, 0, 0, 0), T(0, 0, 0, 0), nul) == 0


def test_usp_auto_select_matches_the_rule(rm):
    from oracle import usp as ousp
    for hkv in (1, 2, 3, 4, 8, 16):
        for group in (1, 2, 4):
            for world in (1, 2, 4, 6, 8, 12, 16, 32):
                assert rm.usp_auto_select(hkv * group, hkv, world) == ousp.auto_select(
                    hkv * group, hkv, world)
    assert rm.usp_auto_select(64, 16, 32, node_size=8) == (8, 4)


def test_usp_auto_select_hand_table(rm):
    from tests.test_oracle_usp import SELECTOR_TABLE
    for (hq, hkv, world, node), want in SELECTOR_TABLE:
        assert rm.usp_auto_select(hq, hkv, world, node_size=node) == want


@pytest.mark.parametrize("kw,u", [(dict(), 3), (dict(), 16), (dict(N=16386, P=2), 4),
                                  (dict(Hq=12, Hkv=6), 4),
                                  (dict(cu_seqlens=16, num_segments=2, B=2), 2)])  # packing: B == 1
def test_usp_validation(rm, kw, u):
    n = ctypes.c_size_t(0)
    d = _desc(rm, **kw)
    assert rm.raw().rm_usp_workspace_size(ctypes.byref(d), u, 0, ctypes.byref(n)) != 0


@pytest.mark.parametrize("kw", [dict(seq_lens=16), dict(cu_seqlens=16, num_segments=3)])
def test_usp_accepts_segments(rm, kw):
    """Packed (B == 1) and right-padded batches under USP: the inner ring sees
    B x u batch entries that share the caller's segment description."""
    n = ctypes.c_size_t(0)
    d = _desc(rm, **kw)
    for backward in (0, 1):
        assert rm.raw().rm_usp_workspace_size(ctypes.byref(d), 2, backward, ctypes.byref(n)) == 0


def test_usp_workspace_sizes(rm):
    n = ctypes.c_size_t(0)
    d = _desc(rm)  # bf16 B=1 Hq=16 Hkv=8 d=128 N=16384 P=2
    q_bytes = 16384 * 16 * 128 * 2
    kv_bytes = 16384 * 8 * 128 * 2
    assert rm.raw().rm_usp_workspace_size(ctypes.byref(d), 2, 0, ctypes.byref(n)) == 0
    assert n.value == 2 * q_bytes + 2 * kv_bytes
    assert rm.raw().rm_usp_workspace_size(ctypes.byref(d), 2, 1, ctypes.byref(n)) == 0
    assert n.value == 4 * q_bytes + 4 * kv_bytes + 16 * 16384 * 4


@pytest.mark.parametrize("gq,gk,status", [(0, 1, 1), (2, 0, 1), (3, 1, 1), (2, 3, 1), (2, 17, 2)])
def test_mesh2d_validation(rm, gq, gk, status):
    n = ctypes.c_size_t(0)
    d = _desc(rm)  # N = 16384
    assert rm.raw().rm_mesh2d_workspace_size(ctypes.byref(d), gq, gk, 0, ctypes.byref(n)) == status
    assert rm.raw().rm_last_error()
    d = _desc(rm, seq_lens=16)  # right-padded (and packed) batches are accepted
    assert rm.raw().rm_mesh2d_workspace_size(ctypes.byref(d), 2, 2, 0, ctypes.byref(n)) == 0


def test_mesh2d_workspace_sizes(rm):
    n = ctypes.c_size_t(0)
    d = _desc(rm)  # bf16 B=1 Hq=16 Hkv=8 d=128 N=16384; P and layout are ignored
    o_slot, lse_slot = 16384 * 16 * 128 * 4, 16384 * 16 * 4
    assert rm.raw().rm_mesh2d_workspace_size(ctypes.byref(d), 4, 8, 0, ctypes.byref(n)) == 0
    assert n.value == 8 * o_slot + 8 * lse_slot
    assert rm.raw().rm_mesh2d_workspace_size(ctypes.byref(d), 4, 8, 1, ctypes.byref(n)) == 0
    assert n.value == lse_slot + o_slot + 2 * (16384 * 8 * 128 * 4)


def test_call_workspace_is_held_and_recorded(rm):
    """A workspace the binding allocates is referenced by the call's holder
    (so it outlives the library call that queues kernels on it), a caller's
    large-enough tensor is used as given, and the tensor is recorded on a
    stream the caller names (not on the current one)."""
    w = rm._Workspace(0, "cpu", None)
    assert w.tensor is None and w.nbytes == 0 and not w.ptr.value
    w = rm._Workspace(64, "cpu", None)
    assert w.tensor is not None and w.nbytes == 64 and w.ptr.value == w.tensor.data_ptr()

    class Caller:
        def __init__(self, n):
            self.buf, self.streams = torch.empty(n, dtype=torch.uint8), []

        def numel(self):
            return self.buf.numel()

        def element_size(self):
            return 1

        def data_ptr(self):
            return self.buf.data_ptr()

        def record_stream(self, s):
            self.streams.append(s)

    mine = Caller(128)
    w = rm._Workspace(100, "cpu", mine)
    assert w.tensor is mine and w.nbytes == 128
    w.done(None)
    assert mine.streams == []
    w.done("side stream")
    assert mine.streams == ["side stream"]
    small = Caller(8)
    assert rm._Workspace(100, "cpu", small).tensor is not small  # too small: one of its own
