"""Thin Python binding of librm_attn.so (argument marshalling only).

Every function here turns torch tensors into the plain pointers, sizes and
strides of the C ABI in ``include/rm_attn.h`` and calls the entry point of the
same name on the current CUDA stream; all computation happens in the CUDA
kernels behind that ABI.  Importing this module loads the library and raises
if it is missing -- there is no CPU fallback.
"""

from __future__ import annotations

import ctypes
import os
from typing import Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "librm_attn.so")

# ---- enums (mirror include/rm_attn.h) ----------------------------------------
RM_OK, RM_ERR_INVALID_ARG, RM_ERR_UNSUPPORTED, RM_ERR_WORKSPACE, RM_ERR_CUDA, RM_ERR_TIMEOUT = range(6)
RM_F32, RM_BF16 = 0, 1
LAYOUTS = {"contiguous": 0, "zigzag": 1, "striped": 2}
MODES = {"fused": 0, "stepwise": 1}
ORDERS = {"rank": 0, "global": 1}

EXPORTED = (
    "rm_attn_block_fwd", "rm_attn_block_bwd", "rm_attn_bwd_preprocess", "rm_lse_merge",
    "rm_ring_workspace_size", "rm_ring_attn_fwd", "rm_ring_attn_bwd", "rm_layout_permute",
    "rm_seq_head_repack", "rm_get_device_status", "rm_status_string", "rm_last_error",
    "rm_debug_expire_wait", "rm_debug_exp2_poly", "rm_ring_attn_bwd_noalloc", "rm_profile_enable", "rm_profile_count",
    "rm_profile_get", "rm_usp_auto_select", "rm_usp_workspace_size", "rm_usp_attn_fwd",
    "rm_usp_attn_bwd", "rm_mesh2d_workspace_size", "rm_mesh2d_attn_fwd", "rm_mesh2d_attn_bwd",
    "rm_convert_f32",
)


class RmTensor(ctypes.Structure):
    _fields_ = [("ptr", ctypes.c_void_p), ("stride_b", ctypes.c_int64),
                ("stride_n", ctypes.c_int64), ("stride_h", ctypes.c_int64)]


class RmAttnDesc(ctypes.Structure):
    _fields_ = [("dtype", ctypes.c_int), ("B", ctypes.c_int), ("Hq", ctypes.c_int),
                ("Hkv", ctypes.c_int), ("d", ctypes.c_int), ("N", ctypes.c_int64),
                ("P", ctypes.c_int), ("layout", ctypes.c_int), ("causal", ctypes.c_int),
                ("scale", ctypes.c_float), ("mode", ctypes.c_int), ("order", ctypes.c_int),
                ("cu_seqlens", ctypes.c_void_p), ("num_segments", ctypes.c_int),
                ("seq_lens", ctypes.c_void_p)]


class RmError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{_status_name(status)}: {msg}")
        self.status = status


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with `python -m sequence_attention_rm_b200.build`")
    lib = ctypes.CDLL(path)
    vp, i, i64, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
    T, D = RmTensor, ctypes.POINTER(RmAttnDesc)
    fp = ctypes.POINTER(ctypes.c_float)
    sig = {
        "rm_attn_block_fwd": [D, i, i, T, T, T, T, i, vp, vp],
        "rm_attn_block_bwd": [D, i, i, T, T, T, T, vp, vp, T, T, T, vp],
        "rm_attn_bwd_preprocess": [i, i, i64, i, i, T, T, vp, vp],
        "rm_convert_f32": [i, i, i64, i, i, T, T, vp],
        "rm_lse_merge": [i, i, i, i64, i, i, ctypes.POINTER(RmTensor), ctypes.POINTER(vp), T, vp, vp],
        "rm_ring_workspace_size": [D, i, ctypes.POINTER(sz)],
        "rm_ring_attn_fwd": [D, T, T, T, T, vp, vp, sz, vp],
        "rm_ring_attn_bwd": [D, T, T, T, T, vp, T, T, T, T, vp, sz, vp],
        "rm_layout_permute": [i, i, i64, i, i, i, i, i, vp, vp, vp],
        "rm_seq_head_repack": [i, i, i64, i, i, i, vp, vp, vp],
        "rm_get_device_status": [vp],
        "rm_debug_expire_wait": [ctypes.c_uint32, vp],
        "rm_debug_exp2_poly": [vp, vp, i64, vp],
        "rm_ring_attn_bwd_noalloc": [D, T, T, T, T, vp, T, T, T, T, vp],
        "rm_profile_enable": [i],
        "rm_profile_count": [],
        "rm_profile_get": [i, ctypes.POINTER(ctypes.c_char_p), ctypes.POINTER(ctypes.c_float)],
        "rm_usp_auto_select": [i, i, i, i, ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_int)],
        "rm_usp_workspace_size": [D, i, i, ctypes.POINTER(sz)],
        "rm_usp_attn_fwd": [D, i, T, T, T, T, vp, vp, sz, vp],
        "rm_usp_attn_bwd": [D, i, T, T, T, T, vp, T, T, T, T, vp, sz, vp],
        "rm_mesh2d_workspace_size": [D, i, i, i, ctypes.POINTER(sz)],
        "rm_mesh2d_attn_fwd": [D, i, i, T, T, T, T, vp, vp, sz, vp],
        "rm_mesh2d_attn_bwd": [D, i, i, T, T, T, T, vp, T, T, T, T, vp, sz, vp],
    }
    for name, args in sig.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = ctypes.c_int
    lib.rm_status_string.argtypes = [ctypes.c_int]
    lib.rm_status_string.restype = ctypes.c_char_p
    lib.rm_last_error.argtypes = []
    lib.rm_last_error.restype = ctypes.c_char_p
    del fp
    return lib


_lib = load_library()


def _status_name(s: int) -> str:
    return _lib.rm_status_string(s).decode()


def _check(status: int) -> None:
    if status != RM_OK:
        raise RmError(status, _lib.rm_last_error().decode())


def _dtype_code(t: torch.dtype) -> int:
    if t == torch.bfloat16:
        return RM_BF16
    if t == torch.float32:
        return RM_F32
    raise TypeError(f"unsupported dtype {t}")


def _stream(stream=None) -> ctypes.c_void_p:
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t: torch.Tensor | None) -> ctypes.c_void_p:
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _bnhd(t: torch.Tensor) -> RmTensor:
    """A [B, N, H, d] tensor with unit stride along d."""
    if t.dim() != 4 or (t.shape[-1] > 1 and t.stride(-1) != 1):
        raise ValueError("expected a [B, N, H, d] tensor with contiguous d")
    return RmTensor(t.data_ptr(), t.stride(0), t.stride(1), t.stride(2))


def _segs(t: torch.Tensor | None):
    if t is None:
        return None
    if t.dtype != torch.int32 or not t.is_cuda or not t.is_contiguous():
        raise ValueError("cu_seqlens / seq_lens must be contiguous CUDA int32 tensors")
    return t.data_ptr()


def desc(dtype: torch.dtype, B: int, Hq: int, Hkv: int, d: int, N: int, P: int, layout: str,
         causal: bool, scale: float | None = None, mode: str = "fused", order: str = "rank",
         cu_seqlens: torch.Tensor | None = None, seq_lens: torch.Tensor | None = None
         ) -> RmAttnDesc:
    """cu_seqlens: packing boundaries (global positions, int32 on the device,
    B == 1); seq_lens: right-padding lengths per batch entry (int32 on the
    device).  The tensors must outlive the asynchronous calls that use them."""
    return RmAttnDesc(_dtype_code(dtype), B, Hq, Hkv, d, N, P, LAYOUTS[layout], int(bool(causal)),
                      0.0 if scale is None else float(scale), MODES[mode], ORDERS[order],
                      _segs(cu_seqlens), 0 if cu_seqlens is None else cu_seqlens.numel() - 1,
                      _segs(seq_lens))


# ---- entry points -----------------------------------------------------------
def layout_permute(x: torch.Tensor, layout: str, P: int, inverse: bool = False,
                   out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Dense [B, N, H, d]: global order -> rank-major (inverse: back)."""
    if not x.is_contiguous():
        raise ValueError("layout_permute needs a dense tensor")
    out = torch.empty_like(x) if out is None else out
    B, N, H, d = x.shape
    _check(_lib.rm_layout_permute(_dtype_code(x.dtype), B, N, H, d, LAYOUTS[layout], P,
                                  int(inverse), _ptr(x), _ptr(out), _stream(stream)))
    return out


def seq_head_repack(x: torch.Tensor, P: int, head_to_seq: bool = False,
                    out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """seq->head: [P, L, H, d] -> [P, P*L, H/P, d]; head->seq is the inverse."""
    if not x.is_contiguous() or x.dim() != 4:
        raise ValueError("seq_head_repack needs a dense 4-d tensor")
    if not head_to_seq:
        _, L, H, d = x.shape
        shape = (P, P * L, H // P, d)
    else:
        _, NL, HP, d = x.shape
        L, H = NL // P, HP * P
        shape = (P, L, H, d)
    out = torch.empty(shape, dtype=x.dtype, device=x.device) if out is None else out
    _check(_lib.rm_seq_head_repack(_dtype_code(x.dtype), P, L, H, d, int(head_to_seq), _ptr(x),
                                   _ptr(out), _stream(stream)))
    return out


def lse_merge(o_parts: Sequence[torch.Tensor], lse_parts: Sequence[torch.Tensor],
              out_dtype: torch.dtype = torch.bfloat16, out: torch.Tensor | None = None,
              lse_out: torch.Tensor | None = None, stream=None):
    """Merge fp32 partials [B, Nq, H, d] with LSE [B, H, Nq] -> (O, LSE)."""
    n = len(o_parts)
    B, Nq, H, d = o_parts[0].shape
    parts = (RmTensor * n)(*[_bnhd(o) for o in o_parts])
    lses = (ctypes.c_void_p * n)(*[l.data_ptr() for l in lse_parts])
    out = torch.empty((B, Nq, H, d), dtype=out_dtype, device=o_parts[0].device) if out is None else out
    lse_out = torch.empty((B, H, Nq), dtype=torch.float32, device=o_parts[0].device) \
        if lse_out is None else lse_out
    _check(_lib.rm_lse_merge(_dtype_code(out_dtype), B, H, Nq, d, n, parts, lses, _bnhd(out),
                             _ptr(lse_out), _stream(stream)))
    return out, lse_out


def attn_block_fwd(q, k, v, *, N: int, P: int, layout: str, causal: bool, q_rank: int,
                   kv_rank: int, scale: float | None = None, o_f32: bool = False, out=None,
                   lse=None, stream=None, cu_seqlens=None, seq_lens=None):
    """One Q shard [B, L, Hq, d] against one KV shard [B, L, Hkv, d] -> (O, LSE)."""
    B, L, Hq, d = q.shape
    dsc = desc(q.dtype, B, Hq, k.shape[2], d, N, P, layout, causal, scale,
               cu_seqlens=cu_seqlens, seq_lens=seq_lens)
    odt = torch.float32 if (o_f32 or q.dtype == torch.float32) else q.dtype
    out = torch.empty((B, L, Hq, d), dtype=odt, device=q.device) if out is None else out
    lse = torch.empty((B, Hq, L), dtype=torch.float32, device=q.device) if lse is None else lse
    _check(_lib.rm_attn_block_fwd(ctypes.byref(dsc), q_rank, kv_rank, _bnhd(q), _bnhd(k), _bnhd(v),
                                  _bnhd(out), int(o_f32), _ptr(lse), _stream(stream)))
    return out, lse


def attn_block_bwd(q, k, v, dout, lse_final, delta, dq_acc, dk_acc, dv_acc, *, N: int, P: int,
                   layout: str, causal: bool, q_rank: int, kv_rank: int,
                   scale: float | None = None, stream=None, cu_seqlens=None, seq_lens=None):
    """Accumulate one shard pair's gradients into fp32 dq_acc / dk_acc / dv_acc."""
    B, L, Hq, d = q.shape
    dsc = desc(q.dtype, B, Hq, k.shape[2], d, N, P, layout, causal, scale,
               cu_seqlens=cu_seqlens, seq_lens=seq_lens)
    _check(_lib.rm_attn_block_bwd(ctypes.byref(dsc), q_rank, kv_rank, _bnhd(q), _bnhd(k), _bnhd(v),
                                  _bnhd(dout), _ptr(lse_final), _ptr(delta), _bnhd(dq_acc),
                                  _bnhd(dk_acc), _bnhd(dv_acc), _stream(stream)))


def convert_f32(x: torch.Tensor, dtype: torch.dtype, out: torch.Tensor | None = None,
                stream=None) -> torch.Tensor:
    """fp32 [B, N, H, d] -> dtype (bf16: round to nearest even)."""
    if x.dtype != torch.float32:
        raise TypeError("convert_f32 takes an fp32 tensor")
    B, N, H, d = x.shape
    out = torch.empty(x.shape, dtype=dtype, device=x.device) if out is None else out
    _check(_lib.rm_convert_f32(_dtype_code(dtype), B, N, H, d, _bnhd(x), _bnhd(out),
                               _stream(stream)))
    return out


def attn_bwd_preprocess(o, dout, delta=None, stream=None):
    """delta [B, H, N] = rowsum(dout * o) in fp32."""
    B, N, H, d = o.shape
    delta = torch.empty((B, H, N), dtype=torch.float32, device=o.device) if delta is None else delta
    _check(_lib.rm_attn_bwd_preprocess(_dtype_code(o.dtype), B, N, H, d, _bnhd(o), _bnhd(dout),
                                       _ptr(delta), _stream(stream)))
    return delta


def ring_workspace_size(dsc: RmAttnDesc, backward: bool) -> int:
    n = ctypes.c_size_t(0)
    _check(_lib.rm_ring_workspace_size(ctypes.byref(dsc), int(backward), ctypes.byref(n)))
    return n.value


class _Workspace:
    """The workspace of one call: the caller's tensor or one allocated here,
    held until the call has queued its kernels.  A tensor allocated here is
    only referenced through this object, so the allocator could hand its
    memory to another allocation (another thread's, or one on another
    stream) before the kernels that use it are queued if it were dropped
    earlier; on a stream other than the current one it is also recorded on
    that stream, so that its memory is not reused before that stream's work
    is done."""

    def __init__(self, nbytes: int, device, ws: torch.Tensor | None):
        if nbytes == 0:
            self.tensor, self.ptr, self.nbytes = None, ctypes.c_void_p(0), 0
            return
        if ws is None or ws.numel() * ws.element_size() < nbytes:
            ws = torch.empty(nbytes, dtype=torch.uint8, device=device)
        self.tensor = ws
        self.ptr, self.nbytes = ctypes.c_void_p(ws.data_ptr()), ws.numel() * ws.element_size()

    def done(self, stream) -> None:
        """Call after the library call returned (its kernels are queued)."""
        if self.tensor is not None and stream is not None:
            self.tensor.record_stream(stream)


def ring_attn_fwd(q, k, v, *, P: int, layout: str, causal: bool, scale: float | None = None,
                  mode: str = "fused", order: str = "rank", cu_seqlens=None, seq_lens=None,
                  out=None, lse=None, ws=None, stream=None):
    """Ring forward over P virtual ranks; q/k/v [B, N, H, d] in `order` ("rank":
    rank-major, "global": the tokens' own order) -> (O, LSE [B, Hq, N]) in the
    same order."""
    B, N, Hq, d = q.shape
    dsc = desc(q.dtype, B, Hq, k.shape[2], d, N, P, layout, causal, scale, mode, order,
               cu_seqlens, seq_lens)
    out = torch.empty_like(q, memory_format=torch.contiguous_format) if out is None else out
    lse = torch.empty((B, Hq, N), dtype=torch.float32, device=q.device) if lse is None else lse
    w = _Workspace(ring_workspace_size(dsc, False), q.device, ws)
    _check(_lib.rm_ring_attn_fwd(ctypes.byref(dsc), _bnhd(q), _bnhd(k), _bnhd(v), _bnhd(out),
                                 _ptr(lse), w.ptr, w.nbytes, _stream(stream)))
    w.done(stream)
    return out, lse


def ring_attn_bwd(q, k, v, o, lse, dout, *, P: int, layout: str, causal: bool,
                  scale: float | None = None, order: str = "rank", cu_seqlens=None,
                  seq_lens=None, dq=None, dk=None, dv=None, ws=None, stream=None):
    """Ring backward; returns (dq, dk, dv) in the input dtype and in `order`."""
    B, N, Hq, d = q.shape
    dsc = desc(q.dtype, B, Hq, k.shape[2], d, N, P, layout, causal, scale, order=order,
               cu_seqlens=cu_seqlens, seq_lens=seq_lens)
    dq = torch.empty_like(q, memory_format=torch.contiguous_format) if dq is None else dq
    dk = torch.empty_like(k, memory_format=torch.contiguous_format) if dk is None else dk
    dv = torch.empty_like(v, memory_format=torch.contiguous_format) if dv is None else dv
    w = _Workspace(ring_workspace_size(dsc, True), q.device, ws)
    _check(_lib.rm_ring_attn_bwd(ctypes.byref(dsc), _bnhd(q), _bnhd(k), _bnhd(v), _bnhd(o),
                                 _ptr(lse), _bnhd(dout), _bnhd(dq), _bnhd(dk), _bnhd(dv), w.ptr, w.nbytes,
                                 _stream(stream)))
    w.done(stream)
    return dq, dk, dv


def ring_attn_bwd_noalloc(q, k, v, o, lse, dout, *, P: int, layout: str, causal: bool,
                          scale: float | None = None, order: str = "rank", dq=None, dk=None,
                          dv=None, stream=None):
    """rm_ring_attn_bwd without a workspace: the library's fixed device scratch
    (at most 64 MiB of workspace) is used instead."""
    B, N, Hq, d = q.shape
    dsc = desc(q.dtype, B, Hq, k.shape[2], d, N, P, layout, causal, scale, order=order)
    dq = torch.empty_like(q, memory_format=torch.contiguous_format) if dq is None else dq
    dk = torch.empty_like(k, memory_format=torch.contiguous_format) if dk is None else dk
    dv = torch.empty_like(v, memory_format=torch.contiguous_format) if dv is None else dv
    _check(_lib.rm_ring_attn_bwd_noalloc(ctypes.byref(dsc), _bnhd(q), _bnhd(k), _bnhd(v), _bnhd(o),
                                         _ptr(lse), _bnhd(dout), _bnhd(dq), _bnhd(dk), _bnhd(dv),
                                         _stream(stream)))
    return dq, dk, dv


def usp_auto_select(Hq: int, Hkv: int, world: int, node_size: int = 8) -> tuple[int, int]:
    """(ulysses, ring) split of `world` virtual devices for USP."""
    u, r = ctypes.c_int(0), ctypes.c_int(0)
    _check(_lib.rm_usp_auto_select(Hq, Hkv, world, node_size, ctypes.byref(u), ctypes.byref(r)))
    return u.value, r.value


def usp_workspace_size(dsc: RmAttnDesc, ulysses: int, backward: bool) -> int:
    n = ctypes.c_size_t(0)
    _check(_lib.rm_usp_workspace_size(ctypes.byref(dsc), ulysses, int(backward), ctypes.byref(n)))
    return n.value


def usp_attn_fwd(q, k, v, *, P: int, ulysses: int, layout: str, causal: bool,
                 scale: float | None = None, mode: str = "fused", order: str = "rank",
                 cu_seqlens=None, seq_lens=None, out=None, lse=None, ws=None, stream=None):
    """USP forward: Ulysses degree `ulysses` x ring degree P; dense q/k/v
    [B, N, H, d] in `order` for the P ring ranks -> (O, LSE [B, Hq, N])."""
    B, N, Hq, d = q.shape
    dsc = desc(q.dtype, B, Hq, k.shape[2], d, N, P, layout, causal, scale, mode, order,
               cu_seqlens, seq_lens)
    out = torch.empty_like(q, memory_format=torch.contiguous_format) if out is None else out
    lse = torch.empty((B, Hq, N), dtype=torch.float32, device=q.device) if lse is None else lse
    w = _Workspace(usp_workspace_size(dsc, ulysses, False), q.device, ws)
    _check(_lib.rm_usp_attn_fwd(ctypes.byref(dsc), ulysses, _bnhd(q), _bnhd(k), _bnhd(v),
                                _bnhd(out), _ptr(lse), w.ptr, w.nbytes, _stream(stream)))
    w.done(stream)
    return out, lse


def usp_attn_bwd(q, k, v, o, lse, dout, *, P: int, ulysses: int, layout: str, causal: bool,
                 scale: float | None = None, order: str = "rank", cu_seqlens=None,
                 seq_lens=None, dq=None, dk=None, dv=None, ws=None, stream=None):
    """USP backward -> (dq, dk, dv) in the input dtype and order."""
    B, N, Hq, d = q.shape
    dsc = desc(q.dtype, B, Hq, k.shape[2], d, N, P, layout, causal, scale, order=order,
               cu_seqlens=cu_seqlens, seq_lens=seq_lens)
    dq = torch.empty_like(q, memory_format=torch.contiguous_format) if dq is None else dq
    dk = torch.empty_like(k, memory_format=torch.contiguous_format) if dk is None else dk
    dv = torch.empty_like(v, memory_format=torch.contiguous_format) if dv is None else dv
    w = _Workspace(usp_workspace_size(dsc, ulysses, True), q.device, ws)
    _check(_lib.rm_usp_attn_bwd(ctypes.byref(dsc), ulysses, _bnhd(q), _bnhd(k), _bnhd(v), _bnhd(o),
                                _ptr(lse), _bnhd(dout), _bnhd(dq), _bnhd(dk), _bnhd(dv), w.ptr, w.nbytes,
                                _stream(stream)))
    w.done(stream)
    return dq, dk, dv


def mesh2d_workspace_size(dsc: RmAttnDesc, grid_q: int, grid_k: int, backward: bool) -> int:
    n = ctypes.c_size_t(0)
    _check(_lib.rm_mesh2d_workspace_size(ctypes.byref(dsc), grid_q, grid_k, int(backward),
                                         ctypes.byref(n)))
    return n.value


def mesh2d_attn_fwd(q, k, v, *, grid_q: int, grid_k: int, causal: bool,
                    scale: float | None = None, cu_seqlens=None, seq_lens=None, out=None,
                    lse=None, ws=None, stream=None):
    """Mesh2D forward over a grid_q x grid_k grid of (query chunk, key chunk)
    tiles; q/k/v [B, N, H, d] in token order -> (O, LSE [B, Hq, N])."""
    B, N, Hq, d = q.shape
    dsc = desc(q.dtype, B, Hq, k.shape[2], d, N, grid_q, "contiguous", causal, scale,
               cu_seqlens=cu_seqlens, seq_lens=seq_lens)
    out = torch.empty_like(q, memory_format=torch.contiguous_format) if out is None else out
    lse = torch.empty((B, Hq, N), dtype=torch.float32, device=q.device) if lse is None else lse
    w = _Workspace(mesh2d_workspace_size(dsc, grid_q, grid_k, False), q.device, ws)
    _check(_lib.rm_mesh2d_attn_fwd(ctypes.byref(dsc), grid_q, grid_k, _bnhd(q), _bnhd(k),
                                   _bnhd(v), _bnhd(out), _ptr(lse), w.ptr, w.nbytes, _stream(stream)))
    w.done(stream)
    return out, lse


def mesh2d_attn_bwd(q, k, v, o, lse, dout, *, grid_q: int, grid_k: int, causal: bool,
                    scale: float | None = None, cu_seqlens=None, seq_lens=None, dq=None,
                    dk=None, dv=None, ws=None, stream=None):
    """Mesh2D backward -> (dq, dk, dv) in the input dtype."""
    B, N, Hq, d = q.shape
    dsc = desc(q.dtype, B, Hq, k.shape[2], d, N, grid_q, "contiguous", causal, scale,
               cu_seqlens=cu_seqlens, seq_lens=seq_lens)
    dq = torch.empty_like(q, memory_format=torch.contiguous_format) if dq is None else dq
    dk = torch.empty_like(k, memory_format=torch.contiguous_format) if dk is None else dk
    dv = torch.empty_like(v, memory_format=torch.contiguous_format) if dv is None else dv
    w = _Workspace(mesh2d_workspace_size(dsc, grid_q, grid_k, True), q.device, ws)
    _check(_lib.rm_mesh2d_attn_bwd(ctypes.byref(dsc), grid_q, grid_k, _bnhd(q), _bnhd(k),
                                   _bnhd(v), _bnhd(o), _ptr(lse), _bnhd(dout), _bnhd(dq),
                                   _bnhd(dk), _bnhd(dv), w.ptr, w.nbytes, _stream(stream)))
    w.done(stream)
    return dq, dk, dv


def get_device_status(stream=None) -> int:
    """Synchronise and return (and clear) the device status word as an rm_status."""
    return _lib.rm_get_device_status(_stream(stream))


def debug_expire_wait(spin_limit: int, stream=None) -> None:
    _check(_lib.rm_debug_expire_wait(spin_limit, _stream(stream)))


def debug_exp2_poly(x: torch.Tensor, stream=None) -> torch.Tensor:
    """The forward's FMA-pipe 2^x on a contiguous fp32 CUDA tensor (test hook)."""
    if x.dtype != torch.float32 or not x.is_cuda or not x.is_contiguous():
        raise ValueError("debug_exp2_poly needs a contiguous fp32 CUDA tensor")
    y = torch.empty_like(x)
    _check(_lib.rm_debug_exp2_poly(_ptr(x), _ptr(y), x.numel(), _stream(stream)))
    return y


def profile_enable(on: bool) -> None:
    """Start (clearing earlier records) or stop per-launch event timing."""
    _check(_lib.rm_profile_enable(int(on)))


def profile_records():
    """[(kernel name, device ms)] of the launches recorded since enabling."""
    out = []
    for i in range(_lib.rm_profile_count()):
        name = ctypes.c_char_p()
        ms = ctypes.c_float()
        _check(_lib.rm_profile_get(i, ctypes.byref(name), ctypes.byref(ms)))
        out.append((name.value.decode(), ms.value))
    return out


def raw():
    """The loaded ctypes library (for tests that call the C ABI directly)."""
    return _lib
