"""Thin ctypes binding over libvsa.so (the C ABI declared in include/vsa.h).

Argument marshalling only: torch allocates device memory for outputs and
workspaces and supplies the current CUDA stream; every step of the VSA
forward runs in the library's CUDA kernels.  There is no CPU fallback: if the
shared library is missing or a call fails, these functions raise.
"""

from __future__ import annotations

import ctypes
import math
import os

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libvsa.so")

VSA_OK = 0
VSA_MAX_BLOCKS = 2048
STATUS_NAMES = {
    0: "VSA_OK", 1: "VSA_ERR_INVALID_ARG", 2: "VSA_ERR_SHAPE", 3: "VSA_ERR_UNSUPPORTED",
    4: "VSA_ERR_CUDA", 5: "VSA_ERR_DEVICE_TIMEOUT", 6: "VSA_ERR_INDEX_RANGE",
    7: "VSA_ERR_WORKSPACE", 8: "VSA_ERR_BLOCK_SIZE",
}

_c_void_p = ctypes.c_void_p
_c_int = ctypes.c_int
_c_int64 = ctypes.c_int64
_c_size_t = ctypes.c_size_t
_c_float = ctypes.c_float
_P32 = ctypes.POINTER(ctypes.c_int32)
_P64 = ctypes.POINTER(ctypes.c_int64)


class VsaStrides(ctypes.Structure):
    """vsa_strides: element strides over (batch, head, sequence slot)."""
    _fields_ = [("batch", ctypes.c_int64), ("head", ctypes.c_int64), ("seq", ctypes.c_int64)]


class VsaLayout(ctypes.Structure):
    """vsa_layout: the strides of q, k, v, out and the gate of one call."""
    _fields_ = [("q", VsaStrides), ("k", VsaStrides), ("v", VsaStrides), ("out", VsaStrides),
                ("gate", VsaStrides)]


_PL = ctypes.POINTER(VsaLayout)
VSA_LAYOUT_BHSD, VSA_LAYOUT_BSHD = 0, 1

# name -> (restype, argtypes); mirrors include/vsa.h
SIGNATURES = {
    "vsa_status_string": (ctypes.c_char_p, [_c_int]),
    "vsa_abi_version": (_c_int, []),
    "vsa_get_device_status": (_c_int, [_c_void_p]),
    "vsa_forward_workspace_size": (_c_size_t, [_c_int] * 5),
    "vsa_forward": (_c_int, [_c_void_p] * 4 + [_c_void_p, _c_void_p] + [_c_int] * 6 +
                    [_c_float, _c_void_p, _c_void_p, _c_void_p, _c_int, _c_void_p, _c_void_p,
                     _c_size_t, _c_void_p]),
    "vsa_make_layout": (_c_int, [_c_int] * 6 + [_PL]),
    "vsa_forward_strided": (_c_int, [_c_void_p] * 4 + [_PL, _c_void_p, _c_void_p] + [_c_int] * 7 +
                            [_c_float, _c_void_p, _c_void_p, _c_void_p, _c_int, _c_void_p,
                             _c_void_p, _c_size_t, _c_void_p]),
    "vsa_forward_bshd": (_c_int, [_c_void_p] * 4 + [_c_void_p, _c_void_p] + [_c_int] * 6 +
                         [_c_float, _c_void_p, _c_void_p, _c_void_p, _c_int, _c_void_p, _c_void_p,
                          _c_size_t, _c_void_p]),
    "vsa_forward_noalloc": (_c_int, [_c_void_p] * 4 + [_c_void_p, _c_void_p] + [_c_int] * 6 +
                            [_c_float, _c_void_p, _c_void_p, _c_void_p, _c_int, _c_void_p,
                             _c_void_p]),
    "vsa_forward_host_workspace_size": (_c_size_t, [_c_int] * 8),
    "vsa_forward_host": (_c_int, [_c_void_p] * 4 + [_c_void_p, _c_void_p] + [_c_int] * 6 +
                         [_c_float, _c_void_p, _c_void_p, _c_void_p, _c_int, _c_void_p, _c_int,
                          _c_void_p, _c_size_t, _c_void_p]),
    "block_sparse_attn_from_indices_workspace_size": (_c_size_t, [_c_int] * 4),
    "block_sparse_attn_from_indices": (_c_int, [_c_void_p] * 7 + [_c_int] * 7 +
                                       [_c_float, _c_void_p, _c_void_p, _PL, _c_void_p, _c_size_t,
                                        _c_void_p]),
    "block_sparse_attn": (_c_int, [_c_void_p] * 6 + [_c_int] * 6 +
                          [_c_float, _c_void_p, _c_void_p, _c_void_p, _PL, _c_void_p, _c_size_t,
                           _c_void_p]),
    "block_sparse_attn_varlen_workspace_size": (_c_size_t, [_c_int] * 4),
    "block_sparse_attn_backward_workspace_size": (_c_size_t, [_c_int] * 4),
    "block_sparse_attn_backward": (_c_int, [_c_void_p] * 10 + [_c_int] * 6 +
                                   [_c_float, _c_void_p, _c_void_p, _c_void_p, _c_void_p,
                                    _c_size_t, _c_void_p]),
    "block_sparse_attn_backward_ex_workspace_size": (_c_size_t, [_c_int] * 6),
    "block_sparse_attn_backward_ex": (_c_int, [_c_void_p] * 10 + [_c_int] * 7 +
                                      [_c_float, _c_void_p, _c_void_p, _c_void_p, _c_void_p,
                                       _c_size_t, _c_void_p]),
    "block_sparse_attn_varlen_backward_workspace_size": (_c_size_t, [_c_int] * 5),
    "block_sparse_attn_varlen_backward": (_c_int, [_c_void_p] * 6 + [_P32] * 6 + [_c_int] * 3 +
                                          [_c_void_p, _c_void_p, _c_int, _c_float, _c_void_p,
                                           _c_void_p, _c_void_p, _c_void_p, _c_size_t,
                                           _c_void_p]),
    "block_sparse_attn_varlen": (_c_int, [_c_void_p] * 3 + [_P32, _P32, _P32, _P32, _P32, _P32] +
                                 [_c_int] * 3 + [_c_void_p, _c_void_p, _c_int, _c_float,
                                                 _c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_void_p,
                                                 _c_void_p, _c_size_t, _c_void_p]),
    "build_vsa_metadata": (_c_int, [_c_int] * 6 + [_P64, _P64, _P32, _P64, _P64, _P32]),
    "vsa_gather_tokens": (_c_int, [_c_void_p, _c_void_p, _c_void_p, _c_int64, _c_int64, _c_int64,
                                   _c_int, _c_void_p]),
    "vsa_scatter_tokens": (_c_int, [_c_void_p, _c_void_p, _c_void_p, _c_int64, _c_int64,
                                    _c_int64, _c_int, _c_void_p]),
    "vsa_selftest_umma": (_c_int, [_c_int, _c_int, _c_void_p, _c_void_p, _c_void_p, _c_void_p]),
    "vsa_selftest_exp2": (_c_int, [_c_void_p, _c_void_p, _c_int64, _c_void_p, _c_void_p]),
    "vsa_permute_rows": (_c_int, [_c_void_p, _c_void_p, _P64, _P64, _c_int, _c_void_p]),
    "vsa_set_profile_events": (_c_int, [ctypes.POINTER(_c_void_p)]),
}

_LIB = None


class VSAError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} failed: {STATUS_NAMES.get(code, code)}")
        self.code = code


def lib() -> ctypes.CDLL:
    """Load libvsa.so (built in-tree); raise if it is missing."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: run `python -m block_sparse_attention_15_b200.build`")
        h = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(h, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = h
    return _LIB


def _check(fn: str, code: int):
    if code != VSA_OK:
        raise VSAError(fn, code)


def _ptr(t):
    return None if t is None else _c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return _c_void_p(s.cuda_stream)


def _require(t, dtype, name, device=True):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if device and not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _require_view(t, name):
    """A bf16 CUDA tensor whose last (head-dim) axis is contiguous and whose
    other strides are multiples of 8 elements (any layout: BHSD, BSHD, a
    slice of a fused tensor, a transposed view)."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != torch.bfloat16:
        raise TypeError(f"{name} must be torch.bfloat16, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dim() != 4 or t.stride(3) != 1:
        raise ValueError(f"{name} must be a 4-D view with a contiguous last axis")
    for ax in range(3):
        if t.shape[ax] > 1 and (t.stride(ax) <= 0 or t.stride(ax) % 8):
            raise ValueError(f"{name}: stride {t.stride(ax)} of axis {ax} is not a positive "
                             "multiple of 8 elements")
    if t.data_ptr() % 16:
        raise ValueError(f"{name} must start on a 16-byte boundary")


def _strides_bhsd(t):
    """vsa_strides of a [B, H, S, D] view."""
    return VsaStrides(t.stride(0), t.stride(1), t.stride(2))


def _layout(q, k, v, out, gate_bshd=None):
    """vsa_layout of [B, H, S, D] views q, k, v, out and a [B, S, H, D] gate."""
    g = (VsaStrides(gate_bshd.stride(0), gate_bshd.stride(2), gate_bshd.stride(1))
         if gate_bshd is not None else VsaStrides(0, 0, 0))
    return VsaLayout(_strides_bhsd(q), _strides_bhsd(k), _strides_bhsd(v), _strides_bhsd(out), g)


def _block_sizes_tensor(bs, n, device):
    if bs is None:
        return None
    if not isinstance(bs, torch.Tensor):
        bs = torch.tensor(list(bs), dtype=torch.int32)
    bs = bs.to(device=device, dtype=torch.int32).contiguous()
    if bs.numel() != n:
        raise ValueError(f"expected {n} block sizes, got {bs.numel()}")
    return bs


def get_device_status(stream=None) -> int:
    """Synchronise the stream, then read and clear the device status word."""
    return lib().vsa_get_device_status(_stream(stream))


def check_device_status(stream=None):
    code = get_device_status(stream)
    if code != VSA_OK:
        raise VSAError("device status", code)


def vsa_forward(q, k, v, gate=None, q_block_sizes=None, kv_block_sizes=None, *, topk: int,
                scale: float | None = None, idx_stride: int | None = None, out=None,
                return_out_c: bool = False, return_pooled: bool = False, workspace=None,
                block: int = 64, stream=None):
    """Full VSA forward through ``vsa_forward_strided`` (see include/vsa.h).

    q: [B, H, Sq_pad, D] bf16; k, v: [B, H, Skv_pad, D]; gate: [B, Sq_pad, H, D]
    or None.  Any of them may be a strided view (head dim contiguous, other
    strides multiples of 8): a BSHD tensor transposed to [B, H, S, D], a
    slice of a fused QKV tensor.  ``out`` (allocated like q if None) may be a
    view too.  ``block``: slots per block, 64, 128 or 256 (VSA-128 / VSA-256
    tiles; S is then padded to multiples of the block).  Returns ``(out, q2k_idx, q2k_num)`` plus
    ``out_c`` and the pooled (qc, kc, vc) when asked.
    """
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _require_view(t, n)
    B, H, Sq, D = q.shape
    Skv = k.shape[2]
    if k.shape != (B, H, Skv, D) or v.shape != k.shape:
        raise ValueError("k and v must be [B, H, Skv_pad, D] matching q")
    if gate is not None:
        _require_view(gate, "gate")
        if gate.shape != (B, Sq, H, D):
            raise ValueError(f"gate must be [B, Sq_pad, H, D] = {(B, Sq, H, D)}, got {tuple(gate.shape)}")
    nq, nkv = Sq // block, Skv // block
    k_eff = min(int(topk), nkv)
    stride = k_eff if idx_stride is None else int(idx_stride)
    dev = q.device
    qbs = _block_sizes_tensor(q_block_sizes, nq, dev)
    kbs = _block_sizes_tensor(kv_block_sizes, nkv, dev)
    if out is None:
        out = torch.empty_like(q)
    _require_view(out, "out")
    if out.shape != q.shape:
        raise ValueError("out must be shaped like q")
    q2k_idx = torch.empty((B, H, nq, stride), dtype=torch.int32, device=dev)
    q2k_num = torch.empty((B, H, nq), dtype=torch.int32, device=dev)
    out_c = torch.empty((B, H, nq, D), dtype=torch.float32, device=dev) if return_out_c else None
    L = lib()
    ws_bytes = L.vsa_forward_workspace_size(B, H, nq, nkv, D)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=dev)
    lay = _layout(q, k, v, out, gate)
    _check("vsa_forward_strided", L.vsa_forward_strided(
        _ptr(q), _ptr(k), _ptr(v), _ptr(gate), ctypes.byref(lay), _ptr(qbs), _ptr(kbs), B, H, Sq,
        Skv, D, int(block), int(topk), float(scale) if scale is not None else 0.0, _ptr(out), _ptr(q2k_idx),
        _ptr(q2k_num), stride, _ptr(out_c), _ptr(workspace), workspace.numel(), _stream(stream)))
    res = [out, q2k_idx, q2k_num]
    if return_out_c:
        res.append(out_c)
    if return_pooled:
        res.append(pooled_views(workspace, B, H, nq, nkv, D))
    return tuple(res)


def vsa_forward_host(q, k, v, gate=None, q_block_sizes=None, kv_block_sizes=None, *, topk: int,
                     scale: float | None = None, idx_stride: int | None = None, out=None,
                     return_indices: bool = False, return_out_c: bool = False,
                     heads_per_chunk: int = 0, workspace=None, device=None, stream=None):
    """Full VSA forward on HOST tensors through ``vsa_forward_host`` (see
    include/vsa.h): the library stages chunks of heads onto the GPU, runs the
    forward and copies the results back, overlapping the three.

    q, k, v, gate: CPU bf16 tensors, shapes as in :func:`vsa_forward` (page-locked
    for the copies to overlap).  Returns ``out`` (a page-locked CPU tensor unless
    ``out`` is given) and, when asked, the host ``q2k_idx``, ``q2k_num`` and
    ``out_c``.  The call is asynchronous on ``stream``; synchronise it before
    reading the results.
    """
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _require(t, torch.bfloat16, n, device=False)
        if t.is_cuda:
            raise ValueError(f"{n} must be a CPU tensor")
    B, H, Sq, D = q.shape
    Skv = k.shape[2]
    if k.shape != (B, H, Skv, D) or v.shape != k.shape:
        raise ValueError("k and v must be [B, H, Skv_pad, D] matching q")
    if gate is not None:
        _require(gate, torch.bfloat16, "gate", device=False)
        if gate.is_cuda or gate.shape != (B, Sq, H, D):
            raise ValueError(f"gate must be a CPU [B, Sq_pad, H, D] = {(B, Sq, H, D)} tensor")
    nq, nkv = Sq // 64, Skv // 64
    k_eff = min(int(topk), nkv)
    stride = k_eff if idx_stride is None else int(idx_stride)
    qbs = None if q_block_sizes is None else torch.tensor(list(q_block_sizes), dtype=torch.int32)
    kbs = None if kv_block_sizes is None else torch.tensor(list(kv_block_sizes), dtype=torch.int32)
    for bs, n, name in ((qbs, nq, "q_block_sizes"), (kbs, nkv, "kv_block_sizes")):
        if bs is not None and bs.numel() != n:
            raise ValueError(f"expected {n} {name}, got {bs.numel()}")
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    if out is None:
        out = torch.empty(q.shape, dtype=torch.bfloat16, pin_memory=True)
    elif out.is_cuda or out.dtype != torch.bfloat16 or out.shape != q.shape or not out.is_contiguous():
        raise ValueError("out must be a contiguous CPU bf16 tensor shaped like q")
    q2k_idx = torch.empty((B, H, nq, stride), dtype=torch.int32, pin_memory=True) if return_indices else None
    q2k_num = torch.empty((B, H, nq), dtype=torch.int32, pin_memory=True) if return_indices else None
    out_c = torch.empty((B, H, nq, D), dtype=torch.float32, pin_memory=True) if return_out_c else None
    L = lib()
    ws_bytes = L.vsa_forward_host_workspace_size(B, H, nq, nkv, D, stride, 1 if gate is not None else 0,
                                                 int(heads_per_chunk))
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=dev)
    with torch.cuda.device(dev):
        _check("vsa_forward_host", L.vsa_forward_host(
            _ptr(q), _ptr(k), _ptr(v), _ptr(gate), _ptr(qbs), _ptr(kbs), B, H, Sq, Skv, D, int(topk),
            float(scale) if scale is not None else 0.0, _ptr(out), _ptr(q2k_idx), _ptr(q2k_num), stride,
            _ptr(out_c), int(heads_per_chunk), _ptr(workspace), workspace.numel(), _stream(stream)))
    res = [out]
    if return_indices:
        res += [q2k_idx, q2k_num]
    if return_out_c:
        res.append(out_c)
    return res[0] if len(res) == 1 else tuple(res)


def pooled_views(workspace, B, H, nq, nkv, D):
    """(qc, kc, vc) fp32 views of a vsa_forward workspace (its documented order)."""
    g = B * H * D * 4

    def a256(x):
        return (x + 255) // 256 * 256

    offs = [0, a256(g * nq), a256(g * nq) + a256(g * nkv)]
    shapes = [(B, H, nq, D), (B, H, nkv, D), (B, H, nkv, D)]
    views = []
    for off, shp in zip(offs, shapes):
        n = int(np.prod(shp))
        views.append(workspace[off:off + 4 * n].view(torch.float32).view(shp))
    return tuple(views)


def _sparse_common(q, k, v, out):
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _require_view(t, n)
    B, H, Sq, D = q.shape
    Skv = k.shape[2]
    if k.shape != (B, H, Skv, D) or v.shape != k.shape:
        raise ValueError("k and v must be [B, H, Skv_pad, D] matching q")
    if out is None:
        out = torch.empty_like(q)
    _require_view(out, "out")
    if out.shape != q.shape:
        raise ValueError("out must be shaped like q")
    return B, H, Sq, Skv, D, out


def block_sparse_attn_from_indices(q, k, v, q2k_idx, q2k_num, q_block_sizes=None,
                                   kv_block_sizes=None, *, scale: float | None = None, out=None,
                                   logit_bound: bool = True, block: int = 64,
                                   return_lse: bool = False, stream=None):
    """Block-sparse attention over the listed tiles (``block_sparse_attn_from_indices``).

    q, k, v, out: [B, H, S, D] views (see :func:`vsa_forward`).  With
    ``logit_bound`` (default) a workspace is passed, so the library bounds
    each query block's logits first and the kernel skips its running-max
    check where the bound allows (same results).  With ``return_lse`` also
    returns the fp32 [B, H, Sq] natural-log log-sum-exp per query row (the
    normaliser :func:`block_sparse_attn_backward` takes)."""
    B, H, Sq, Skv, D, out = _sparse_common(q, k, v, out)
    _require(q2k_idx, torch.int32, "q2k_idx")
    _require(q2k_num, torch.int32, "q2k_num")
    nq, nkv = Sq // block, Skv // block
    if q2k_idx.dim() != 4 or q2k_idx.shape[:3] != (B, H, nq) or q2k_num.shape != (B, H, nq):
        raise ValueError("q2k_idx must be [B, H, n_q_blocks, stride], q2k_num [B, H, n_q_blocks]")
    dev = q.device
    qbs = _block_sizes_tensor(q_block_sizes, nq, dev)
    kbs = _block_sizes_tensor(kv_block_sizes, nkv, dev)
    L = lib()
    ws = None
    if logit_bound:
        ws = torch.empty(max(L.block_sparse_attn_from_indices_workspace_size(B, H, nq, nkv), 256),
                         dtype=torch.uint8, device=dev)
    lay = _layout(q, k, v, out)
    lse = torch.empty((B, H, Sq), dtype=torch.float32, device=dev) if return_lse else None
    _check("block_sparse_attn_from_indices", L.block_sparse_attn_from_indices(
        _ptr(q), _ptr(k), _ptr(v), _ptr(q2k_idx), _ptr(q2k_num), _ptr(qbs), _ptr(kbs), B, H, Sq,
        Skv, D, int(block), q2k_idx.shape[3], float(scale) if scale is not None else 0.0, _ptr(out),
        _ptr(lse), ctypes.byref(lay), _ptr(ws), 0 if ws is None else ws.numel(), _stream(stream)))
    return (out, lse) if return_lse else out


def block_sparse_attn(q, k, v, block_map, q_block_sizes=None, kv_block_sizes=None, *,
                      scale: float | None = None, out=None, return_indices: bool = False,
                      block: int = 64, stream=None):
    """Block-sparse attention from a bool block map [B, H, n_q_blocks,
    n_kv_blocks] (``block_sparse_attn``): converted on the device to index
    rows, then the index-native kernel.  With ``return_indices`` also
    returns the (q2k_idx, q2k_num) it produced."""
    B, H, Sq, Skv, D, out = _sparse_common(q, k, v, out)
    nq, nkv = Sq // block, Skv // block
    if not isinstance(block_map, torch.Tensor) or block_map.dtype != torch.bool:
        raise TypeError("block_map must be a torch.bool tensor")
    if tuple(block_map.shape) != (B, H, nq, nkv) or not block_map.is_cuda or not block_map.is_contiguous():
        raise ValueError(f"block_map must be a contiguous CUDA [B, H, n_q_blocks, n_kv_blocks] = "
                         f"{(B, H, nq, nkv)} tensor")
    dev = q.device
    qbs = _block_sizes_tensor(q_block_sizes, nq, dev)
    kbs = _block_sizes_tensor(kv_block_sizes, nkv, dev)
    q2k_idx = torch.empty((B, H, nq, nkv), dtype=torch.int32, device=dev)
    q2k_num = torch.empty((B, H, nq), dtype=torch.int32, device=dev)
    L = lib()
    ws = torch.empty(max(L.block_sparse_attn_from_indices_workspace_size(B, H, nq, nkv), 256),
                     dtype=torch.uint8, device=dev)
    lay = _layout(q, k, v, out)
    _check("block_sparse_attn", L.block_sparse_attn(
        _ptr(q), _ptr(k), _ptr(v), _ptr(block_map), _ptr(qbs), _ptr(kbs), B, H, Sq, Skv, D,
        int(block), float(scale) if scale is not None else 0.0, _ptr(out), _ptr(q2k_idx), _ptr(q2k_num),
        ctypes.byref(lay), _ptr(ws), ws.numel(), _stream(stream)))
    return (out, q2k_idx, q2k_num) if return_indices else out


def video_sparse_attn_bshd(q, k, v, gate=None, q_block_sizes=None, kv_block_sizes=None, *,
                           topk: int, scale: float | None = None, idx_stride: int | None = None,
                           out=None, return_out_c: bool = False, workspace=None, block: int = 64,
                           stream=None):
    """The whole VSA forward on BSHD tensors: q [B, Sq_pad, H, D], k and v
    [B, Skv_pad, H, D], gate [B, Sq_pad, H, D]; the output is BSHD too.  The
    library reads and writes the BSHD memory in place (strided views, no
    transposed copies).  Returns ``(out, q2k_idx, q2k_num)`` (+ ``out_c``)."""
    if out is None and isinstance(q, torch.Tensor):
        out = torch.empty_like(q)
    res = vsa_forward(q.transpose(1, 2), k.transpose(1, 2), v.transpose(1, 2), gate,
                      q_block_sizes, kv_block_sizes, topk=topk, scale=scale, idx_stride=idx_stride,
                      out=None if out is None else out.transpose(1, 2), return_out_c=return_out_c,
                      workspace=workspace, block=block, stream=stream)
    return (out,) + tuple(res[1:])


def block_sparse_attn_backward(q, k, v, out, dout, lse, q2k_idx, q2k_num, q_block_sizes=None,
                               kv_block_sizes=None, *, scale: float | None = None, block: int = 64,
                               stream=None):
    """dq, dk, dv of :func:`block_sparse_attn_from_indices` (contiguous BHSD)
    for the output gradient ``dout``; ``out`` and ``lse`` come from that
    forward call (``return_lse=True``), ``block`` is its block size.  Block
    64 calls ``block_sparse_attn_backward``; 128 and 256 call
    ``block_sparse_attn_backward_ex``, which rewrites the selection over
    64-slot sub-blocks on the device first."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (out, "out"), (dout, "dout")):
        _require(t, torch.bfloat16, n)
    _require(lse, torch.float32, "lse")
    _require(q2k_idx, torch.int32, "q2k_idx")
    _require(q2k_num, torch.int32, "q2k_num")
    B, H, Sq, D = q.shape
    Skv = k.shape[2]
    nq, nkv = Sq // block, Skv // block
    if out.shape != q.shape or dout.shape != q.shape or lse.shape != (B, H, Sq):
        raise ValueError("out and dout must be shaped like q, lse [B, H, Sq_pad]")
    if q2k_idx.dim() != 4 or q2k_idx.shape[:3] != (B, H, nq) or q2k_num.shape != (B, H, nq):
        raise ValueError("q2k_idx must be [B, H, n_q_blocks, stride], q2k_num [B, H, n_q_blocks]")
    dev = q.device
    qbs = _block_sizes_tensor(q_block_sizes, nq, dev)
    kbs = _block_sizes_tensor(kv_block_sizes, nkv, dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    L = lib()
    sc = float(scale) if scale is not None else 0.0
    width = q2k_idx.shape[3]
    if block == 64:
        ws = torch.empty(max(L.block_sparse_attn_backward_workspace_size(B, H, Sq, nkv), 256),
                         dtype=torch.uint8, device=dev)
        _check("block_sparse_attn_backward", L.block_sparse_attn_backward(
            _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(dout), _ptr(lse), _ptr(q2k_idx),
            _ptr(q2k_num), _ptr(qbs), _ptr(kbs), B, H, Sq, Skv, D, width, sc, _ptr(dq), _ptr(dk),
            _ptr(dv), _ptr(ws), ws.numel(), _stream(stream)))
        return dq, dk, dv
    need = L.block_sparse_attn_backward_ex_workspace_size(B, H, Sq, Skv, int(block), width)
    ws = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    _check("block_sparse_attn_backward_ex", L.block_sparse_attn_backward_ex(
        _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(dout), _ptr(lse), _ptr(q2k_idx), _ptr(q2k_num),
        _ptr(qbs), _ptr(kbs), B, H, Sq, Skv, D, int(block), width, sc, _ptr(dq), _ptr(dk), _ptr(dv),
        _ptr(ws), ws.numel(), _stream(stream)))
    return dq, dk, dv


def _host_i32(xs):
    arr = np.ascontiguousarray(np.asarray(xs, dtype=np.int32))
    return arr, arr.ctypes.data_as(_P32)


def block_sparse_attn_varlen(q, k, v, cu_seqlens_q, cu_seqlens_kv, q2k_idx, q2k_num, *,
                             scale: float | None = None, q_block_sizes_list=None,
                             kv_block_sizes_list=None, return_aux: bool = False, out=None,
                             lse=None, stream=None):
    """Varlen block-sparse attention (``block_sparse_attn_varlen``).

    q: [H, total_q, D]; k, v: [H, total_kv, D]; cu_seqlens_*: host sequences
    of n+1 ints; q2k_idx: [H, total_q_blocks, stride] with per-sequence local
    indices.  With ``return_aux`` also returns (pack_index_q, pack_index_kv,
    q2k_idx_rebased).
    """
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _require(t, torch.bfloat16, n)
    _require(q2k_idx, torch.int32, "q2k_idx")
    _require(q2k_num, torch.int32, "q2k_num")
    H, total_q, D = q.shape
    cq, cq_p = _host_i32(cu_seqlens_q)
    ck, ck_p = _host_i32(cu_seqlens_kv)
    n = len(cq) - 1
    keep = [cq, ck]

    def sizes(lst):
        if lst is None:
            return None, None, None
        flat = [int(s) for seq in lst for s in seq]
        cub = [0]
        for seq in lst:
            cub.append(cub[-1] + len(seq))
        a, ap = _host_i32(flat)
        b, bp = _host_i32(cub)
        keep.extend([a, b])
        return ap, bp, len(flat)

    qs_p, qcb_p, nqb = sizes(q_block_sizes_list)
    ks_p, kcb_p, nkb = sizes(kv_block_sizes_list)
    if nqb is None:
        nqb = sum(-(-(int(cq[i + 1]) - int(cq[i])) // 64) for i in range(n))
    if nkb is None:
        nkb = sum(-(-(int(ck[i + 1]) - int(ck[i])) // 64) for i in range(n))
    dev = q.device
    if out is None:
        out = torch.zeros_like(q)
    L = lib()
    ws_bytes = L.block_sparse_attn_varlen_workspace_size(max(n, 1), max(nqb, 1), max(nkb, 1), max(H, 1))
    ws = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=dev)
    aux = None
    if return_aux:
        aux = (torch.empty(64 * nqb, dtype=torch.int64, device=dev),
               torch.empty(64 * nkb, dtype=torch.int64, device=dev),
               torch.empty_like(q2k_idx))
    stride = q2k_idx.shape[-1]
    _check("block_sparse_attn_varlen", L.block_sparse_attn_varlen(
        _ptr(q), _ptr(k), _ptr(v), cq_p, ck_p, qs_p, qcb_p, ks_p, kcb_p, n, H, D, _ptr(q2k_idx),
        _ptr(q2k_num), stride, float(scale) if scale is not None else 0.0, _ptr(out), _ptr(lse),
        _ptr(aux[0]) if aux else None, _ptr(aux[1]) if aux else None,
        _ptr(aux[2]) if aux else None, _ptr(ws), ws.numel(), _stream(stream)))
    del keep
    return (out, *aux) if return_aux else out


def block_sparse_attn_varlen_backward(q, k, v, out, dout, lse, cu_seqlens_q, cu_seqlens_kv,
                                      q2k_idx, q2k_num, *, scale: float | None = None,
                                      stream=None):
    """dq, dk, dv of :func:`block_sparse_attn_varlen` (64-token blocks with a
    partial last block per sequence); ``out`` and ``lse`` [H, total_q] come
    from that forward call."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (out, "out"), (dout, "dout")):
        _require(t, torch.bfloat16, n)
    _require(lse, torch.float32, "lse")
    _require(q2k_idx, torch.int32, "q2k_idx")
    _require(q2k_num, torch.int32, "q2k_num")
    H, total_q, D = q.shape
    cq, cq_p = _host_i32(cu_seqlens_q)
    ck, ck_p = _host_i32(cu_seqlens_kv)
    n = len(cq) - 1
    nqb = sum(-(-(int(cq[i + 1]) - int(cq[i])) // 64) for i in range(n))
    nkb = sum(-(-(int(ck[i + 1]) - int(ck[i])) // 64) for i in range(n))
    dq, dk, dv = torch.zeros_like(q), torch.zeros_like(k), torch.zeros_like(v)
    L = lib()
    ws = torch.empty(max(L.block_sparse_attn_varlen_backward_workspace_size(n, nqb, nkb, H, total_q), 256),
                     dtype=torch.uint8, device=q.device)
    _check("block_sparse_attn_varlen_backward", L.block_sparse_attn_varlen_backward(
        _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(dout), _ptr(lse), cq_p, ck_p, None, None, None,
        None, n, H, D, _ptr(q2k_idx), _ptr(q2k_num), q2k_idx.shape[-1],
        float(scale) if scale is not None else 0.0, _ptr(dq), _ptr(dk), _ptr(dv), _ptr(ws),
        ws.numel(), _stream(stream)))
    del cq, ck
    return dq, dk, dv


def build_vsa_metadata(T: int, Hh: int, W: int, tile=(4, 4, 4)) -> dict:
    """Tile metadata from the library's host routine (numpy arrays)."""
    L = lib()
    n_tiles = ctypes.c_int32(0)
    _check("build_vsa_metadata", L.build_vsa_metadata(T, Hh, W, *tile, None, None, None, None, None,
                                                      ctypes.byref(n_tiles)))
    N = T * Hh * W
    vol = int(np.prod(tile))
    nt = n_tiles.value
    perm = np.empty(N, dtype=np.int64)
    rev = np.empty(N, dtype=np.int64)
    vbs = np.empty(nt, dtype=np.int32)
    npi = np.empty(N, dtype=np.int64)
    slot = np.empty(nt * vol, dtype=np.int64)
    _check("build_vsa_metadata", L.build_vsa_metadata(
        T, Hh, W, *tile, perm.ctypes.data_as(_P64), rev.ctypes.data_as(_P64),
        vbs.ctypes.data_as(_P32), npi.ctypes.data_as(_P64), slot.ctypes.data_as(_P64),
        ctypes.byref(n_tiles)))
    return dict(tile_partition_indices=perm, reverse_tile_partition_indices=rev,
                variable_block_sizes=vbs, non_pad_index=npi, slot_token=slot, n_tiles=nt,
                max_block_size=vol)


def gather_tokens(x, slot_token, *, stream=None):
    """[G, N, D] tokens -> [G, n_slots, D] padded block layout (zeros in pads)."""
    _require(x, torch.bfloat16, "x")
    _require(slot_token, torch.int64, "slot_token")
    G, N, D = x.shape
    ns = slot_token.numel()
    dst = torch.empty((G, ns, D), dtype=x.dtype, device=x.device)
    _check("vsa_gather_tokens", lib().vsa_gather_tokens(_ptr(x), _ptr(dst), _ptr(slot_token), N, ns,
                                                        G, D, _stream(stream)))
    return dst


def scatter_tokens(x_pad, slot_token, n_tokens: int, *, stream=None):
    """Inverse of :func:`gather_tokens` on the real tokens."""
    _require(x_pad, torch.bfloat16, "x_pad")
    _require(slot_token, torch.int64, "slot_token")
    G, ns, D = x_pad.shape
    dst = torch.empty((G, n_tokens, D), dtype=x_pad.dtype, device=x_pad.device)
    _check("vsa_scatter_tokens", lib().vsa_scatter_tokens(_ptr(x_pad), _ptr(dst), _ptr(slot_token),
                                                          n_tokens, ns, G, D, _stream(stream)))
    return dst


def selftest_umma(mode: int, a, b, *, stream=None):
    """Run one tensor-core product of the sparse kernel on global operands."""
    _require(a, torch.bfloat16, "a")
    _require(b, torch.bfloat16, "b")
    D = b.shape[1] if mode >= 2 else a.shape[1]
    shape = {0: (128, 64), 1: (D, 64), 2: (128, 128), 3: (128, D)}[mode]
    c = torch.empty(shape, dtype=torch.float32, device=a.device)
    _check("vsa_selftest_umma", lib().vsa_selftest_umma(mode, D, _ptr(a), _ptr(b), _ptr(c),
                                                        _stream(stream)))
    return c


def permute_rows(src, extents, src_strides, *, out=None, stream=None):
    """``vsa_permute_rows``: rows of the last axis of ``src`` (a contiguous
    bf16 CUDA tensor, D = src.shape[-1]) gathered into a new tensor of shape
    (*extents, D): out[a0, a1, a2, a3] = src row a0*S0 + a1*S1 + a2*S2 + a3*S3."""
    _require(src, torch.bfloat16, "src")
    D = src.shape[-1]
    ext = [int(e) for e in extents]
    st = [int(x) for x in src_strides]
    if len(ext) != 4 or len(st) != 4:
        raise ValueError("extents and src_strides take four entries")
    rows = src.numel() // D
    if any(e > 0 for e in ext) and sum((e - 1) * s_ for e, s_ in zip(ext, st) if e > 0) >= rows:
        raise ValueError("the strides reach past the end of src")
    if out is None:
        out = torch.empty((*ext, D), dtype=src.dtype, device=src.device)
    _require(out, torch.bfloat16, "out")
    e64 = (ctypes.c_int64 * 4)(*ext)
    s64 = (ctypes.c_int64 * 4)(*st)
    _check("vsa_permute_rows", lib().vsa_permute_rows(_ptr(src), _ptr(out), e64, s64, D,
                                                      _stream(stream)))
    return out


def selftest_exp2(x, *, stream=None):
    """The sparse kernel's FMA-pipe 2^x on a device fp32 tensor; returns
    (y, number of elements whose packed halves disagree)."""
    _require(x, torch.float32, "x")
    y = torch.empty_like(x)
    mism = torch.zeros(1, dtype=torch.int32, device=x.device)
    _check("vsa_selftest_exp2", lib().vsa_selftest_exp2(_ptr(x), _ptr(y), x.numel(), _ptr(mism),
                                                        _stream(stream)))
    return y, int(mism.item())


def set_profile_events(events):
    """Record four torch.cuda.Event objects around vsa_forward's kernels
    (before pool, after pool, after coarse/top-k, after block-sparse), or
    switch the hook off with None."""
    if events is None:
        _check("vsa_set_profile_events", lib().vsa_set_profile_events(None))
        return
    for e in events:
        if not e.cuda_event:  # torch creates the handle on first record
            e.record()
    arr = (_c_void_p * 4)(*[e.cuda_event for e in events])
    _check("vsa_set_profile_events", lib().vsa_set_profile_events(arr))


def default_scale(D: int) -> float:
    return 1.0 / math.sqrt(D)
