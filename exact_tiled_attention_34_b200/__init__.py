"""Exact tiled attention on B200 (sm_100a): thin Python binding of libfa.so.

Every function here only marshals torch tensors into the C ABI declared in
``include/fa.h``; all arithmetic runs in the library's CUDA kernels. PyTorch is
used for device memory and streams only. There is no fallback: if the library
is missing or a tensor is not a CUDA tensor, the call raises.

    o, lse = forward(q, k, v, causal=False, scale=None)
    o, lse = forward_blocksparse(q, k, v, tile_mask, scale=None)
    dq, dk, dv = backward(q, k, v, o, lse, do, causal=False, scale=None)
    dq, dk, dv = backward_blocksparse(q, k, v, o, lse, do, tile_mask, scale=None)

Tensors are bf16 contiguous on one CUDA device: q, o, do [B, H, Nq, d]; k, v
[B, H, Nk, d]; lse fp32 [B, H, Nq]. Nq and Nk may differ (then the causal mask is
bottom-right aligned: query i sees key j iff j <= i + Nk - Nq); the block-sparse
calls need Nq = Nk = N and a uint8 tile_mask [ceil(N/128), ceil(N/128)]. Any N >= 1,
d in {64, 96, 128}. forward/backward/attention also take layout="bnhd" for [B, N, H, d]
tensors (lse stays [B, H, Nq]).
"""
from __future__ import annotations

import ctypes
import math
import os
import re

__all__ = [
    "FAError", "lib", "lib_path", "exported_names", "forward", "forward_blocksparse", "backward",
    "backward_blocksparse", "bwd_workspace_bytes", "device_status", "STATUS", "bwd_preprocess", "bwd_dkdv",
    "bwd_dq", "bwd_fused_preprocess", "bwd_fused_main", "bwd_fused_dq", "attention", "attention_blocksparse", "forward_dropout", "backward_dropout", "merge_partial",
    "accumulate_bf16", "to_bf16", "forward_merge", "bwd_fused_main_f32", "accumulate_f32",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
_HEADER = os.path.join(os.path.dirname(_HERE), "include", "fa.h")

STATUS = {
    0: "FA_OK", 1: "FA_ERR_INVALID_ARG", 2: "FA_ERR_UNSUPPORTED", 3: "FA_ERR_ALIGNMENT",
    4: "FA_ERR_WORKSPACE", 5: "FA_ERR_CUDA", 6: "FA_ERR_DEVICE_TIMEOUT",
}


class FAError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = int(status)
        super().__init__(f"{what}: {STATUS.get(self.status, self.status)}")


def lib_path() -> str:
    return os.environ.get("FA_LIB", os.path.join(_HERE, "libfa.so"))


_lib = None
_vp, _i, _f, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
_u64, _u32 = ctypes.c_uint64, ctypes.c_uint32
_SIGS = {
    "fa_status_string": ([_i], ctypes.c_char_p),
    "fa_version": ([], _i),
    "fa_fwd": ([_vp] * 5 + [_i] * 5 + [_f, _vp], _i),
    "fa_fwd_qk": ([_vp] * 5 + [_i] * 6 + [_f, _vp], _i),
    "fa_fwd_ex": ([_vp] * 5 + [_i] * 7 + [_f, _vp], _i),
    "fa_fwd_blocksparse": ([_vp] * 6 + [_i] * 5 + [_f, _vp], _i),
    "fa_bwd_workspace_bytes": ([_i] * 4, _sz),
    "fa_bwd": ([_vp] * 10 + [_sz] + [_i] * 5 + [_f, _vp], _i),
    "fa_bwd_qk": ([_vp] * 10 + [_sz] + [_i] * 6 + [_f, _vp], _i),
    "fa_bwd_ex": ([_vp] * 10 + [_sz] + [_i] * 7 + [_f, _vp], _i),
    "fa_bwd_blocksparse": ([_vp] * 10 + [_sz, _vp, _i] + [_i] * 4 + [_f, _vp], _i),
    "fa_device_status": ([_vp, ctypes.POINTER(_i)], _i),
    "fa_bwd_preprocess": ([_vp] * 4 + [_sz] + [_i] * 4 + [_vp], _i),
    "fa_bwd_dkdv": ([_vp] * 7 + [_sz, _vp, _i] + [_i] * 5 + [_f, _vp], _i),
    "fa_bwd_dq": ([_vp] * 6 + [_sz, _vp, _i] + [_i] * 5 + [_f, _vp], _i),
    "fa_fwd_dropout": ([_vp] * 5 + [_i] * 5 + [_f, _f, _u64, _u32, _vp], _i),
    "fa_bwd_dropout": ([_vp] * 10 + [_sz] + [_i] * 5 + [_f, _f, _u64, _u32, _vp], _i),
    "fa_merge_partial": ([_vp, _vp, _vp, _vp, ctypes.c_longlong, _i, _vp], _i),
    "fa_accumulate_bf16": ([_vp, _vp, ctypes.c_longlong, _i, _vp], _i),
    "fa_to_bf16": ([_vp, _vp, ctypes.c_longlong, _vp], _i),
    "fa_bwd_fused_workspace_bytes": ([_i] * 4, _sz),
    "fa_bwd_fused": ([_vp] * 10 + [_sz] + [_i] * 5 + [_f, _vp], _i),
    "fa_bwd_fused_ex": ([_vp] * 10 + [_sz, _vp, _i] + [_i] * 7 + [_f, _vp], _i),
    "fa_bwd_fused_preprocess": ([_vp] * 4 + [_sz] + [_i] * 4 + [_vp], _i),
    "fa_bwd_fused_main": ([_vp] * 7 + [_sz, _vp, _i] + [_i] * 5 + [_f, _vp], _i),
    "fa_bwd_fused_dq": ([_vp, _vp, _sz] + [_i] * 4 + [_f, _vp], _i),
    "fa_fwd_merge": ([_vp] * 5 + [_i] * 5 + [_f, _vp], _i),
    "fa_bwd_fused_main_f32": ([_vp] * 7 + [_sz] + [_i] * 5 + [_f, _vp], _i),
    "fa_accumulate_f32": ([_vp, _vp, ctypes.c_longlong, _vp], _i),
    "fa_debug_exp2": ([_vp, _vp, _i, _i, _vp], _i),
    "fa_debug_wait_timeout": ([_i, _vp, _vp], _i),
    "fa_debug_stall_producer": ([_i, _i], _i),
}


def lib():
    """The loaded C library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        path = lib_path()
        if not os.path.exists(path):
            raise FAError(5, f"{path} is missing; build it with `python -m exact_tiled_attention_34_b200.build`")
        handle = ctypes.CDLL(path)
        for name, (args, res) in _SIGS.items():
            fn = getattr(handle, name)
            fn.argtypes = args
            fn.restype = res
        _lib = handle
    return _lib


def exported_names():
    """Function names declared in include/fa.h."""
    with open(_HEADER) as f:
        src = f.read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[\w\s\*]+?\b(fa_\w+)\s*\(", src, re.M)))


def _check(status: int, what: str):
    if status != 0:
        raise FAError(status, what)


def _stream_ptr(dev):
    import torch
    return ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)


_LAYOUTS = {"bhnd": 0, "bnhd": 1}


def _dims(q, k, layout):
    """(B, H, Nq, Nk, d) of q [B, H, Nq, d] / k [B, H, Nk, d] ("bhnd") or q [B, Nq, H, d] /
    k [B, Nk, H, d] ("bnhd")."""
    if layout not in _LAYOUTS:
        raise ValueError(f"layout must be one of {sorted(_LAYOUTS)}")
    if layout == "bhnd":
        return q.shape[0], q.shape[1], q.shape[2], k.shape[2], q.shape[3]
    return q.shape[0], q.shape[2], q.shape[1], k.shape[1], q.shape[3]


def _check_qkv(q, k, v, *qlike, layout="bhnd"):
    """q and the tensors in qlike (o, dO) share a shape; k and v share one; batch, heads
    and head dim agree (in the positions of `layout`)."""
    import torch
    for t in (q, k, v) + qlike:
        if not t.is_cuda:
            raise ValueError("tensors must be CUDA tensors (no CPU path)")
        if t.dtype != torch.bfloat16:
            raise ValueError("q, k, v, o, dO must be bfloat16")
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous [B, H, N, d]")
        if t.device != q.device:
            raise ValueError("all tensors must be on one device")
    if q.dim() != 4 or k.dim() != 4:
        raise ValueError("expected [B, H, N, d] tensors")
    if k.shape != v.shape or any(t.shape != q.shape for t in qlike):
        raise ValueError("k and v must share a shape, as must q, o and dO")
    hq, hk = (1, 1) if layout == "bhnd" else (2, 2)
    if (q.shape[0], q.shape[hq], q.shape[3]) != (k.shape[0], k.shape[hk], k.shape[3]):
        raise ValueError("q and k must agree in batch, heads and head dim")


def _check_buffer(t, shape, dtype, device, what):
    """A caller-supplied output, row array or workspace: contiguous, of `dtype`, on
    `device` and (unless shape is None) of `shape`. The C entry points receive only its
    pointer, so a smaller tensor, or one on another device, would be written or read out
    of bounds by the kernels."""
    if t.dtype != dtype or not t.is_contiguous() or t.device != device:
        raise ValueError(f"{what} must be a contiguous {dtype} tensor on {device}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{what} must have shape {tuple(shape)}, not {tuple(t.shape)}")


def _check_outputs(q, out, lse, rows):
    """out like q (bf16) and lse fp32 [B, H, Nq] (`rows`), where the caller supplies them."""
    import torch
    if out is not None:
        _check_buffer(out, q.shape, torch.bfloat16, q.device, "out")
    if lse is not None:
        _check_buffer(lse, rows, torch.float32, q.device, "lse")


def _check_equal_lengths(q, k, what):
    if tuple(k.shape) != tuple(q.shape):
        raise ValueError(f"{what} needs equal query and key lengths")


def _scale(scale, d):
    return 1.0 / math.sqrt(d) if scale is None else float(scale)


def forward(q, k, v, causal: bool = False, scale=None, out=None, lse=None, layout: str = "bhnd"):
    """O = softmax(scale q k^T [causal]) v and the fp32 row log-sum-exp [B, H, Nq]."""
    import torch
    _check_qkv(q, k, v, layout=layout)
    B, H, N, Nk, d = _dims(q, k, layout)
    _check_outputs(q, out, lse, (B, H, N))
    o = torch.empty_like(q) if out is None else out
    l = torch.empty((B, H, N), dtype=torch.float32, device=q.device) if lse is None else lse
    with torch.cuda.device(q.device):
        if layout != "bhnd":
            st = lib().fa_fwd_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), l.data_ptr(),
                                 B, H, N, Nk, d, _LAYOUTS[layout], int(bool(causal)), _scale(scale, d),
                                 _stream_ptr(q.device))
        elif Nk == N:
            st = lib().fa_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), l.data_ptr(),
                              B, H, N, d, int(bool(causal)), _scale(scale, d), _stream_ptr(q.device))
        else:
            st = lib().fa_fwd_qk(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), l.data_ptr(),
                                 B, H, N, Nk, d, int(bool(causal)), _scale(scale, d), _stream_ptr(q.device))
    _check(st, "fa_fwd")
    return o, l


def _check_mask(tile_mask, q, mask_block):
    import torch
    if tile_mask.dtype != torch.uint8 or not tile_mask.is_contiguous() or tile_mask.device != q.device:
        raise ValueError("tile_mask must be a contiguous uint8 tensor on the device of q")
    nt = -(-q.shape[2] // mask_block)  # ceil: a partial last tile has its own mask entry
    if tuple(tile_mask.shape) != (nt, nt):
        raise ValueError(f"tile_mask must be [{nt}, {nt}]")


def forward_blocksparse(q, k, v, tile_mask, scale=None, mask_block: int = 128, out=None, lse=None):
    """Block-sparse forward: attention restricted to the kept 128x128 tiles."""
    import torch
    _check_qkv(q, k, v)
    _check_equal_lengths(q, k, "block-sparse attention")
    _check_mask(tile_mask, q, mask_block)
    B, H, N, d = q.shape
    _check_outputs(q, out, lse, (B, H, N))
    o = torch.empty_like(q) if out is None else out
    l = torch.empty((B, H, N), dtype=torch.float32, device=q.device) if lse is None else lse
    with torch.cuda.device(q.device):
        st = lib().fa_fwd_blocksparse(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), l.data_ptr(),
                                      tile_mask.data_ptr(), mask_block, B, H, N, d, _scale(scale, d),
                                      _stream_ptr(q.device))
    _check(st, "fa_fwd_blocksparse")
    return o, l


def _seed_args(p, seed, offset):
    p = float(p)
    if not (0.0 <= p < 1.0):
        raise ValueError("dropout probability must be in [0, 1)")
    return p, int(seed) & 0xFFFFFFFFFFFFFFFF, int(offset) & 0xFFFFFFFF


def forward_dropout(q, k, v, p: float, seed: int, offset: int = 0, causal: bool = False, scale=None, out=None,
                    lse=None):
    """Forward with dropout on the attention probabilities (keep mask from Philox,
    seeded by (seed, offset)): O = (P * M * 256/t) V with t = round(256 (1 - p)); lse is
    that of the softmax before dropout. q, k, v [B, H, N, d], d 64 or 128."""
    import torch
    _check_qkv(q, k, v)
    if k.shape != q.shape:
        raise ValueError("dropout needs equal query and key lengths")
    p, seed, offset = _seed_args(p, seed, offset)
    B, H, N, d = q.shape
    _check_outputs(q, out, lse, (B, H, N))
    o = torch.empty_like(q) if out is None else out
    l = torch.empty((B, H, N), dtype=torch.float32, device=q.device) if lse is None else lse
    with torch.cuda.device(q.device):
        st = lib().fa_fwd_dropout(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), l.data_ptr(), B, H, N, d,
                                  int(bool(causal)), _scale(scale, d), p, seed, offset, _stream_ptr(q.device))
    _check(st, "fa_fwd_dropout")
    return o, l


def bwd_workspace_bytes(B: int, H: int, N: int, d: int, deterministic: bool = True) -> int:
    """Workspace bytes of the deterministic backward, or (deterministic=False) of the
    fused backward, which also holds an fp32 dQ accumulator."""
    if deterministic:
        return int(lib().fa_bwd_workspace_bytes(B, H, N, d))
    return int(lib().fa_bwd_fused_workspace_bytes(B, H, N, d))


def _bwd_prep(q, k, v, o, lse, do, workspace, grads, layout="bhnd", deterministic=True):
    import torch
    _check_qkv(q, k, v, o, do, layout=layout)
    B, H, N, _, d = _dims(q, k, layout)
    if lse.dtype != torch.float32 or tuple(lse.shape) != (B, H, N) or not lse.is_contiguous():
        raise ValueError("lse must be contiguous fp32 [B, H, N]")
    need = bwd_workspace_bytes(B, H, N, d, deterministic)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    else:
        _check_buffer(workspace, None, torch.uint8, q.device, "workspace")  # its size is checked in C
    if grads is None:
        grads = (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v))
    else:
        if len(grads) != 3:
            raise ValueError("grads must be (dq, dk, dv)")
        for g, like, name in zip(grads, (q, k, v), ("dq", "dk", "dv")):
            _check_buffer(g, like.shape, torch.bfloat16, q.device, name)
    return workspace, grads


def _bwd_fused(q, k, v, o, lse, do, causal, scale, workspace, grads, layout, tile_mask, mask_block):
    import torch
    workspace, (dq, dk, dv) = _bwd_prep(q, k, v, o, lse, do, workspace, grads, layout, deterministic=False)
    B, H, N, Nk, d = _dims(q, k, layout)
    with torch.cuda.device(q.device):
        st = lib().fa_bwd_fused_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                                   do.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), workspace.data_ptr(),
                                   workspace.numel(), None if tile_mask is None else tile_mask.data_ptr(),
                                   mask_block, B, H, N, Nk, d, _LAYOUTS[layout], int(bool(causal)),
                                   _scale(scale, d), _stream_ptr(q.device))
    _check(st, "fa_bwd_fused_ex")
    return dq, dk, dv


def _deterministic(deterministic, d):
    """The backward to use: True (two-kernel, bit-reproducible) unless asked otherwise;
    head dim 256 has only the fused backward."""
    if deterministic is None:
        return d != 256
    if deterministic and d == 256:
        raise ValueError("head dim 256 has only the fused backward (deterministic=False)")
    return bool(deterministic)


def backward(q, k, v, o, lse, do, causal: bool = False, scale=None, workspace=None, grads=None,
             layout: str = "bhnd", deterministic=None):
    """Gradients (dq, dk, dv) of sum(O * dO) given the forward's o and lse.

    deterministic=True (the default for head dims 64, 96, 128): the two-kernel backward
    (bit-reproducible). False (the default, and only choice, at head dim 256): the fused
    single kernel (five products per tile pair instead of seven; dq accumulated in fp32
    in an order that varies from run to run)."""
    import torch
    if not _deterministic(deterministic, q.shape[-1]):
        return _bwd_fused(q, k, v, o, lse, do, causal, scale, workspace, grads, layout, None, 128)
    workspace, (dq, dk, dv) = _bwd_prep(q, k, v, o, lse, do, workspace, grads, layout)
    B, H, N, Nk, d = _dims(q, k, layout)
    with torch.cuda.device(q.device):
        if layout != "bhnd":
            st = lib().fa_bwd_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                                 do.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), workspace.data_ptr(),
                                 workspace.numel(), B, H, N, Nk, d, _LAYOUTS[layout], int(bool(causal)),
                                 _scale(scale, d), _stream_ptr(q.device))
        elif Nk == N:
            st = lib().fa_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), do.data_ptr(),
                              dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), workspace.data_ptr(), workspace.numel(),
                              B, H, N, d, int(bool(causal)), _scale(scale, d), _stream_ptr(q.device))
        else:
            st = lib().fa_bwd_qk(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                                 do.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), workspace.data_ptr(),
                                 workspace.numel(), B, H, N, Nk, d, int(bool(causal)), _scale(scale, d),
                                 _stream_ptr(q.device))
    _check(st, "fa_bwd")
    return dq, dk, dv


def backward_dropout(q, k, v, o, lse, do, p: float, seed: int, offset: int = 0, causal: bool = False, scale=None,
                     workspace=None, grads=None):
    """Gradients of sum(O * dO) for ``forward_dropout`` with the same p, seed and offset."""
    import torch
    if k.shape != q.shape:
        raise ValueError("dropout needs equal query and key lengths")
    p, seed, offset = _seed_args(p, seed, offset)
    workspace, (dq, dk, dv) = _bwd_prep(q, k, v, o, lse, do, workspace, grads)
    B, H, N, d = q.shape
    with torch.cuda.device(q.device):
        st = lib().fa_bwd_dropout(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                                  do.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), workspace.data_ptr(),
                                  workspace.numel(), B, H, N, d, int(bool(causal)), _scale(scale, d), p, seed,
                                  offset, _stream_ptr(q.device))
    _check(st, "fa_bwd_dropout")
    return dq, dk, dv


def backward_blocksparse(q, k, v, o, lse, do, tile_mask, scale=None, mask_block: int = 128, workspace=None,
                         grads=None, deterministic=None):
    """Block-sparse backward (same mask as the forward); deterministic as for backward."""
    import torch
    _check_qkv(q, k, v, o, do)
    _check_equal_lengths(q, k, "block-sparse attention")
    _check_mask(tile_mask, q, mask_block)
    if not _deterministic(deterministic, q.shape[-1]):
        return _bwd_fused(q, k, v, o, lse, do, False, scale, workspace, grads, "bhnd", tile_mask, mask_block)
    workspace, (dq, dk, dv) = _bwd_prep(q, k, v, o, lse, do, workspace, grads)
    B, H, N, d = q.shape
    with torch.cuda.device(q.device):
        st = lib().fa_bwd_blocksparse(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                                      do.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                                      workspace.data_ptr(), workspace.numel(), tile_mask.data_ptr(), mask_block,
                                      B, H, N, d, _scale(scale, d), _stream_ptr(q.device))
    _check(st, "fa_bwd_blocksparse")
    return dq, dk, dv


def device_status(device=None):
    """Synchronise the current stream and return (status, detail) of the device status word."""
    import torch
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    detail = ctypes.c_int(0)
    with torch.cuda.device(dev):
        st = lib().fa_device_status(_stream_ptr(dev), ctypes.byref(detail))
    return int(st), int(detail.value)


# ---------------------------------------------------------------- staged backward
# The three launches of ``backward`` as separate calls (same workspace for all three).

def _check_stage(q, *like, lse=None, workspace=None, tile_mask=None, mask_block=128):
    """Arguments of a staged call: q and every tensor in `like` contiguous bf16 CUDA
    tensors of q's [B, H, N, d] shape on q's device (one length for queries and keys);
    lse fp32 [B, H, N]; the workspace uint8 on that device (its size is checked in C);
    the tile mask as for the block-sparse calls."""
    import torch
    _check_qkv(q, q, q, *like)
    if lse is not None:
        _check_buffer(lse, q.shape[:3], torch.float32, q.device, "lse")
    if workspace is not None:
        _check_buffer(workspace, None, torch.uint8, q.device, "workspace")
    if tile_mask is not None:
        _check_mask(tile_mask, q, mask_block)

def bwd_preprocess(o, do, lse, workspace):
    import torch
    _check_stage(o, do, lse=lse, workspace=workspace)
    B, H, N, d = o.shape
    with torch.cuda.device(o.device):
        st = lib().fa_bwd_preprocess(o.data_ptr(), do.data_ptr(), lse.data_ptr(), workspace.data_ptr(),
                                     workspace.numel(), B, H, N, d, _stream_ptr(o.device))
    _check(st, "fa_bwd_preprocess")


def bwd_dkdv(q, k, v, do, dk, dv, workspace, causal=False, scale=None, tile_mask=None, mask_block=128):
    import torch
    _check_stage(q, k, v, do, dk, dv, workspace=workspace, tile_mask=tile_mask, mask_block=mask_block)
    B, H, N, d = q.shape
    with torch.cuda.device(q.device):
        st = lib().fa_bwd_dkdv(q.data_ptr(), k.data_ptr(), v.data_ptr(), do.data_ptr(), dk.data_ptr(),
                               dv.data_ptr(), workspace.data_ptr(), workspace.numel(),
                               None if tile_mask is None else tile_mask.data_ptr(), mask_block,
                               B, H, N, d, int(bool(causal)), _scale(scale, d), _stream_ptr(q.device))
    _check(st, "fa_bwd_dkdv")


def bwd_dq(q, k, v, do, dq, workspace, causal=False, scale=None, tile_mask=None, mask_block=128):
    import torch
    _check_stage(q, k, v, do, dq, workspace=workspace, tile_mask=tile_mask, mask_block=mask_block)
    B, H, N, d = q.shape
    with torch.cuda.device(q.device):
        st = lib().fa_bwd_dq(q.data_ptr(), k.data_ptr(), v.data_ptr(), do.data_ptr(), dq.data_ptr(),
                             workspace.data_ptr(), workspace.numel(),
                             None if tile_mask is None else tile_mask.data_ptr(), mask_block,
                             B, H, N, d, int(bool(causal)), _scale(scale, d), _stream_ptr(q.device))
    _check(st, "fa_bwd_dq")


# The three launches of ``backward(..., deterministic=False)`` as separate calls
# (workspace of bwd_workspace_bytes(..., deterministic=False), the same for all three).

def bwd_fused_preprocess(o, do, lse, workspace):
    import torch
    _check_stage(o, do, lse=lse, workspace=workspace)
    B, H, N, d = o.shape
    with torch.cuda.device(o.device):
        st = lib().fa_bwd_fused_preprocess(o.data_ptr(), do.data_ptr(), lse.data_ptr(), workspace.data_ptr(),
                                           workspace.numel(), B, H, N, d, _stream_ptr(o.device))
    _check(st, "fa_bwd_fused_preprocess")


def bwd_fused_main(q, k, v, do, dk, dv, workspace, causal=False, scale=None, tile_mask=None, mask_block=128):
    import torch
    _check_stage(q, k, v, do, dk, dv, workspace=workspace, tile_mask=tile_mask, mask_block=mask_block)
    B, H, N, d = q.shape
    with torch.cuda.device(q.device):
        st = lib().fa_bwd_fused_main(q.data_ptr(), k.data_ptr(), v.data_ptr(), do.data_ptr(), dk.data_ptr(),
                                     dv.data_ptr(), workspace.data_ptr(), workspace.numel(),
                                     None if tile_mask is None else tile_mask.data_ptr(), mask_block,
                                     B, H, N, d, int(bool(causal)), _scale(scale, d), _stream_ptr(q.device))
    _check(st, "fa_bwd_fused_main")


def bwd_fused_dq(dq, workspace, scale=None):
    import torch
    _check_stage(dq, workspace=workspace)
    B, H, N, d = dq.shape
    with torch.cuda.device(dq.device):
        st = lib().fa_bwd_fused_dq(dq.data_ptr(), workspace.data_ptr(), workspace.numel(), B, H, N, d,
                                   _scale(scale, d), _stream_ptr(dq.device))
    _check(st, "fa_bwd_fused_dq")


def debug_exp2(x, mode: int):
    """2^x on the device through one of the kernels' two exponential paths
    (0: special-function unit, 1: the library's polynomial). x: fp32 CUDA tensor."""
    import torch
    if not x.is_cuda or x.dtype != torch.float32 or not x.is_contiguous():
        raise ValueError("x must be a contiguous fp32 CUDA tensor")
    y = torch.empty_like(x)
    with torch.cuda.device(x.device):
        st = lib().fa_debug_exp2(x.data_ptr(), y.data_ptr(), x.numel(), mode, _stream_ptr(x.device))
    _check(st, "fa_debug_exp2")
    return y


def debug_wait_timeout(timeout_us: int, device=None):
    """Run the bounded-wait self-test kernel and return (status, detail, out):
    the status word after it (as device_status) and out = [warp 0 gave up at its
    limit, warp 1 left on the abort flag, warp 0's wait in microseconds]."""
    import torch
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    out = torch.full((3,), -1, dtype=torch.int32, device=dev)
    with torch.cuda.device(dev):
        st = lib().fa_debug_wait_timeout(int(timeout_us), out.data_ptr(), _stream_ptr(dev))
    _check(st, "fa_debug_wait_timeout")
    status, detail = device_status(dev)
    return status, detail, out.tolist()


def debug_stall_producer(on: bool, timeout_us: int = 2000):
    """Test hook: while on, attention launches run with an idle TMA producer and a
    wait limit of timeout_us, so that they end through their timeout path."""
    _check(lib().fa_debug_stall_producer(1 if on else 0, int(timeout_us)), "fa_debug_stall_producer")


# ---------------------------------------------------------------- key-block merging
# Element-wise kernels for attention split over key blocks (see ``ring``).

def merge_partial(o_acc, lse_acc, o_part, lse_part):
    """In place: (o_acc fp32, lse_acc fp32) <- the log-sum-exp merge with one key block's
    partial result (o_part bf16, lse_part fp32), all [B, H, N, d] / [B, H, N]."""
    import torch
    if o_acc.dtype != torch.float32 or o_part.dtype != torch.bfloat16 or o_acc.shape != o_part.shape:
        raise ValueError("o_acc must be fp32 and o_part bf16 of one shape")
    if lse_acc.dtype != torch.float32 or lse_part.dtype != torch.float32 or lse_acc.shape != lse_part.shape:
        raise ValueError("lse_acc and lse_part must be fp32 of one shape")
    # The kernel indexes O at row * d for every lse row: one lse entry per row of O.
    if o_acc.dim() < 1 or tuple(lse_acc.shape) != tuple(o_acc.shape[:-1]):
        raise ValueError("lse_acc must have the shape of o_acc without its last dimension")
    for t in (o_acc, lse_acc, o_part, lse_part):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError("contiguous CUDA tensors expected")
    d = o_acc.shape[-1]
    with torch.cuda.device(o_acc.device):
        st = lib().fa_merge_partial(o_acc.data_ptr(), lse_acc.data_ptr(), o_part.data_ptr(), lse_part.data_ptr(),
                                    lse_acc.numel(), d, _stream_ptr(o_acc.device))
    _check(st, "fa_merge_partial")


def accumulate_bf16(acc, x, overwrite: bool = False):
    """In place: acc (fp32) <- (0 if overwrite else acc) + x (bf16), same shape."""
    import torch
    if acc.dtype != torch.float32 or x.dtype != torch.bfloat16 or acc.shape != x.shape:
        raise ValueError("acc must be fp32 and x bf16 of one shape")
    if not (acc.is_cuda and x.is_cuda and acc.is_contiguous() and x.is_contiguous()):
        raise ValueError("contiguous CUDA tensors expected")
    with torch.cuda.device(acc.device):
        st = lib().fa_accumulate_bf16(acc.data_ptr(), x.data_ptr(), acc.numel(), int(bool(overwrite)),
                                      _stream_ptr(acc.device))
    _check(st, "fa_accumulate_bf16")


def forward_merge(q, k, v, o_acc, lse_acc, causal: bool = False, scale=None):
    """In place: (o_acc fp32 [B, H, N, d], lse_acc fp32 [B, H, N]) <- the running result
    merged with the attention of q against this key block (k, v), in the kernel."""
    import torch
    _check_qkv(q, k, v)
    if k.shape != q.shape:
        raise ValueError("query and key blocks must have the same shape")
    if o_acc.dtype != torch.float32 or tuple(o_acc.shape) != tuple(q.shape) or not o_acc.is_contiguous() \
            or o_acc.device != q.device:
        raise ValueError("o_acc must be a contiguous fp32 tensor of q's shape on q's device")
    if lse_acc.dtype != torch.float32 or tuple(lse_acc.shape) != tuple(q.shape[:3]) or not lse_acc.is_contiguous() \
            or lse_acc.device != q.device:
        raise ValueError("lse_acc must be a contiguous fp32 [B, H, N] tensor on q's device")
    B, H, N, d = q.shape
    with torch.cuda.device(q.device):
        st = lib().fa_fwd_merge(q.data_ptr(), k.data_ptr(), v.data_ptr(), o_acc.data_ptr(), lse_acc.data_ptr(), B, H, N,
                                d, int(bool(causal)), _scale(scale, d), _stream_ptr(q.device))
    _check(st, "fa_fwd_merge")


def bwd_fused_main_f32(q, k, v, do, dk32, dv32, workspace, causal=False, scale=None):
    """The fused backward's main kernel with fp32 dK, dV outputs (dQ's share added into the
    workspace's accumulator, as bwd_fused_main)."""
    import torch
    _check_stage(q, k, v, do, workspace=workspace)
    B, H, N, d = q.shape
    for t in (dk32, dv32):
        if t.dtype != torch.float32 or tuple(t.shape) != tuple(k.shape) or not t.is_contiguous() \
                or t.device != q.device:
            raise ValueError("dk32 and dv32 must be contiguous fp32 tensors of k's shape on q's device")
    with torch.cuda.device(q.device):
        st = lib().fa_bwd_fused_main_f32(q.data_ptr(), k.data_ptr(), v.data_ptr(), do.data_ptr(), dk32.data_ptr(),
                                         dv32.data_ptr(), workspace.data_ptr(), workspace.numel(), B, H, N, d,
                                         int(bool(causal)), _scale(scale, d), _stream_ptr(q.device))
    _check(st, "fa_bwd_fused_main_f32")


def accumulate_f32(acc, x):
    """In place: acc (fp32) += x (fp32), same shape."""
    import torch
    if acc.dtype != torch.float32 or x.dtype != torch.float32 or acc.shape != x.shape:
        raise ValueError("acc and x must be fp32 of one shape")
    if not (acc.is_cuda and x.is_cuda and acc.is_contiguous() and x.is_contiguous()):
        raise ValueError("contiguous CUDA tensors expected")
    with torch.cuda.device(acc.device):
        st = lib().fa_accumulate_f32(acc.data_ptr(), x.data_ptr(), acc.numel(), _stream_ptr(acc.device))
    _check(st, "fa_accumulate_f32")


def to_bf16(x, out=None):
    """bf16 copy of an fp32 CUDA tensor (round to nearest even), through the library."""
    import torch
    if x.dtype != torch.float32 or not x.is_cuda or not x.is_contiguous():
        raise ValueError("x must be a contiguous fp32 CUDA tensor")
    out = torch.empty(x.shape, dtype=torch.bfloat16, device=x.device) if out is None else out
    with torch.cuda.device(x.device):
        st = lib().fa_to_bf16(out.data_ptr(), x.data_ptr(), x.numel(), _stream_ptr(x.device))
    _check(st, "fa_to_bf16")
    return out


# ---------------------------------------------------------------- autograd
# torch.autograd glue around forward/backward: the forward saves q, k, v, o and lse,
# the backward hands them with dO to the library's backward. Marshalling only.

def _autograd_fn():
    import torch

    class _Attention(torch.autograd.Function):
        @staticmethod
        def forward(ctx, q, k, v, causal, scale, tile_mask, layout, drop):
            if drop is not None:
                o, lse = forward_dropout(q, k, v, *drop, causal=causal, scale=scale)
            elif tile_mask is None:
                o, lse = forward(q, k, v, causal=causal, scale=scale, layout=layout)
            else:
                o, lse = forward_blocksparse(q, k, v, tile_mask, scale=scale)
            ctx.save_for_backward(q, k, v, o, lse)
            ctx.causal, ctx.scale, ctx.tile_mask, ctx.layout, ctx.drop = causal, scale, tile_mask, layout, drop
            ctx.mark_non_differentiable(lse)
            return o, lse

        @staticmethod
        def backward(ctx, do, _dlse):
            q, k, v, o, lse = ctx.saved_tensors
            do = do.contiguous()
            if ctx.drop is not None:
                dq, dk, dv = backward_dropout(q, k, v, o, lse, do, *ctx.drop, causal=ctx.causal, scale=ctx.scale)
            elif ctx.tile_mask is None:
                dq, dk, dv = backward(q, k, v, o, lse, do, causal=ctx.causal, scale=ctx.scale, layout=ctx.layout)
            else:
                dq, dk, dv = backward_blocksparse(q, k, v, o, lse, do, ctx.tile_mask, scale=ctx.scale)
            return dq, dk, dv, None, None, None, None, None

    return _Attention


_ATTN = None


def attention(q, k, v, causal: bool = False, scale=None, layout: str = "bhnd", dropout_p: float = 0.0,
              seed=None, offset: int = 0):
    """Differentiable O = softmax(scale q k^T [causal]) v for torch.autograd: the
    forward and backward run in the library (q, k, v and layout as for ``forward``).
    dropout_p > 0 applies dropout to the probabilities (see ``forward_dropout``); the
    seed is drawn from torch's default CPU generator when not given, and the backward
    reuses it."""
    global _ATTN
    if _ATTN is None:
        _ATTN = _autograd_fn()
    drop = None
    if dropout_p:
        if layout != "bhnd":
            raise ValueError("dropout is implemented for the [B, H, N, d] layout")
        if seed is None:
            import torch
            seed = int(torch.randint(0, 2 ** 62, (1,), dtype=torch.int64).item())
        drop = (float(dropout_p), int(seed), int(offset))
    o, _ = _ATTN.apply(q, k, v, bool(causal), scale, None, layout, drop)
    return o


def attention_blocksparse(q, k, v, tile_mask, scale=None):
    """Differentiable block-sparse attention (see ``forward_blocksparse``)."""
    global _ATTN
    if _ATTN is None:
        _ATTN = _autograd_fn()
    o, _ = _ATTN.apply(q, k, v, False, scale, tile_mask, "bhnd", None)
    return o
