"""Python binding of libssta.so, the SSTA forward library for B200 (sm_100a).

Argument marshalling only: every step of the path runs in the library's CUDA
kernels.  The functions carry the C entry points' names (include/ssta.h) and
take torch CUDA tensors, whose device pointers and the current CUDA stream are
passed through.  Output tensors that the caller does not supply are allocated
here with torch (the library itself never allocates).  There is no CPU
fallback: if libssta.so is missing, importing this package raises.
"""
from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass

import torch

__all__ = [
    "SstaError", "SSTA_BF16", "SSTA_F32", "Desc", "desc_from", "ssta_plan", "ssta_tile_reorder",
    "ssta_build_block_mask", "ssta_attention_fwd", "ssta_attention_bwd", "ssta_tile_unorder", "ssta_read_device_status",
    "ssta_status_string", "ssta_forward", "library_path", "lib",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libssta.so")

if not os.path.exists(_LIB_PATH):
    raise ImportError(
        f"{_LIB_PATH} is missing: build it with `python block_sparse_video_ssta_b200/build.py` "
        "(there is no fallback implementation)")

lib = ctypes.CDLL(_LIB_PATH)

SSTA_BF16 = 0
SSTA_F32 = 1
SCORE_MODES = {"similarity": 0, "importance": 1}
COMBINE_MODES = {"union": 0, "and": 1}
WINDOW_MODES = {"shift": 0, "truncate": 1}
_STATUS = {0: "SSTA_OK", 1: "SSTA_ERR_INVALID_ARG", 2: "SSTA_ERR_UNSUPPORTED", 3: "SSTA_ERR_ALIGNMENT",
           4: "SSTA_ERR_WORKSPACE", 5: "SSTA_ERR_LAUNCH", 6: "SSTA_ERR_DEVICE_TIMEOUT",
           7: "SSTA_ERR_DEVICE_BOUNDS"}


class Desc(ctypes.Structure):
    """Mirror of ssta_desc."""
    _fields_ = [(n, ctypes.c_int) for n in
                ("B", "H", "D", "T", "Y", "X", "tT", "tY", "tX", "wT", "wY", "wX", "topk", "L_text", "dtype")] + [
        ("scale", ctypes.c_float), ("score_mode", ctypes.c_int), ("lambda_", ctypes.c_float),
        ("combine", ctypes.c_int), ("window_mode", ctypes.c_int)]


class _PlanInfo(ctypes.Structure):
    _fields_ = [("packed_len", ctypes.c_int64), ("num_tiles", ctypes.c_int), ("num_text_tiles", ctypes.c_int),
                ("num_q_tiles", ctypes.c_int), ("tile_tokens", ctypes.c_int), ("topk", ctypes.c_int),
                ("window_tiles", ctypes.c_int), ("max_kept", ctypes.c_int), ("workspace_bytes", ctypes.c_size_t),
                ("attn_workspace_bytes", ctypes.c_size_t), ("bwd_workspace_bytes", ctypes.c_size_t)]


_P = ctypes.c_void_p
_D = ctypes.POINTER(Desc)
_sig = {
    "ssta_plan": [_D, ctypes.POINTER(_PlanInfo)],
    "ssta_tile_reorder": [_D, _P, _P, _P, _P],
    "ssta_build_block_mask": [_D, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P],
    "ssta_attention_fwd": [_D, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P],
    "ssta_attention_bwd": [_D, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P],
    "ssta_tile_unorder": [_D, _P, _P, _P, _P],
    "ssta_read_device_status": [_P, _P, ctypes.POINTER(ctypes.c_int32)],
}
for _name, _args in _sig.items():
    _f = getattr(lib, _name)
    _f.argtypes = _args
    _f.restype = ctypes.c_int
lib.ssta_status_string.argtypes = [ctypes.c_int]
lib.ssta_status_string.restype = ctypes.c_char_p


class SstaError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {ssta_status_string(code)} ({code})")


def library_path() -> str:
    return _LIB_PATH


def ssta_status_string(code: int) -> str:
    return lib.ssta_status_string(int(code)).decode()


def _check(code: int, where: str):
    if code != 0:
        raise SstaError(code, where)


def desc_from(w=None, **kw) -> Desc:
    """Build a descriptor from any object with the descriptor's field names (e.g. a
    workload), overridden by keyword arguments.  ``dtype`` may be "bf16"/"f32" or
    the enum value; the mask modes ``score_mode`` ("similarity"/"importance"),
    ``combine`` ("union"/"and") and ``window_mode`` ("shift"/"truncate") may be
    names or enum values, and ``lam`` is the importance weight (default 0.9)."""
    fields = {}
    for n in ("B", "H", "D", "T", "Y", "X", "tT", "tY", "tX", "wT", "wY", "wX", "topk", "L_text", "dtype"):
        if n in kw:
            fields[n] = kw[n]
        elif w is not None and hasattr(w, n):
            fields[n] = getattr(w, n)
        else:
            raise ValueError(f"descriptor field {n} missing")
    dt = fields["dtype"]
    if isinstance(dt, str):
        fields["dtype"] = {"bf16": SSTA_BF16, "f32": SSTA_F32}[dt]
    scale = kw.get("scale", getattr(w, "scale", 0.0) if w is not None else 0.0) or 0.0

    def mode(name, table, default):
        v = kw.get(name, getattr(w, name, default) if w is not None else default)
        return table[v] if isinstance(v, str) else int(v)
    lam = float(kw.get("lam", getattr(w, "lam", 0.9) if w is not None else 0.9))
    return Desc(**{k: int(v) for k, v in fields.items()}, scale=float(scale),
                score_mode=mode("score_mode", SCORE_MODES, "similarity"), lambda_=lam,
                combine=mode("combine", COMBINE_MODES, "union"), window_mode=mode("window_mode", WINDOW_MODES, "shift"))


@dataclass
class Plan:
    packed_len: int
    num_tiles: int
    num_text_tiles: int
    num_q_tiles: int
    tile_tokens: int
    topk: int
    window_tiles: int
    max_kept: int
    workspace_bytes: int
    attn_workspace_bytes: int
    bwd_workspace_bytes: int


def ssta_plan(desc: Desc) -> Plan:
    info = _PlanInfo()
    _call("ssta_plan", None, ctypes.byref(desc), ctypes.byref(info))
    return Plan(*(getattr(info, f[0]) for f in _PlanInfo._fields_))


def _torch_dtype(desc: Desc):
    return torch.bfloat16 if desc.dtype == SSTA_BF16 else torch.float32


def _stream(stream, device):
    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _ptr(t, name, dtype=None, shape=None, optional=False):
    if t is None:
        if optional:
            return None
        raise ValueError(f"{name} is required")
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (there is no CPU path)")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    return ctypes.c_void_p(t.data_ptr())


def _call(name, dev, *args):
    """Call C-ABI function `name` with CUDA device `dev` current (the device whose stream
    and tensors the call receives; None for host-only calls); raise on a non-zero status."""
    fn = getattr(lib, name)
    if dev is None:
        return _check(fn(*args), name)
    with torch.cuda.device(dev):
        return _check(fn(*args), name)


def _workspace(nbytes, device):
    # 256-byte aligned (the caching allocator returns 512-byte aligned blocks)
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def ssta_tile_reorder(desc: Desc, x_raster, x_text=None, x_packed=None, stream=None):
    """Step 1: raster [B,H,T,Y,X,D] (+ text [B,H,L,D]) -> packed [B,H,Lq,D]."""
    p = ssta_plan(desc)
    dt = _torch_dtype(desc)
    dev = x_raster.device
    if x_packed is None:
        x_packed = torch.empty((desc.B, desc.H, p.packed_len, desc.D), dtype=dt, device=dev)
    _call(
        "ssta_tile_reorder", dev, ctypes.byref(desc),
        _ptr(x_raster, "x_raster", dt, (desc.B, desc.H, desc.T, desc.Y, desc.X, desc.D)),
        _ptr(x_text, "x_text", dt, (desc.B, desc.H, desc.L_text, desc.D), optional=desc.L_text == 0),
        _ptr(x_packed, "x_packed", dt, (desc.B, desc.H, p.packed_len, desc.D)),
        _stream(stream, dev))
    return x_packed


def ssta_build_block_mask(desc: Desc, q_packed, k_packed, kv_idx=None, kv_cnt=None, tile_scores=None,
                          workspace=None, stream=None):
    """Steps 2-4 (mask): returns (kv_idx [B,H,NQ,max_kept], kv_cnt [B,H,NQ], workspace)."""
    p = ssta_plan(desc)
    dt = _torch_dtype(desc)
    dev = q_packed.device
    shp = (desc.B, desc.H, p.packed_len, desc.D)
    if kv_idx is None:
        kv_idx = torch.empty((desc.B, desc.H, p.num_q_tiles, p.max_kept), dtype=torch.int32, device=dev)
    if kv_cnt is None:
        kv_cnt = torch.empty((desc.B, desc.H, p.num_q_tiles), dtype=torch.int32, device=dev)
    if workspace is None:
        workspace = _workspace(p.workspace_bytes, dev)
    _call(
        "ssta_build_block_mask", dev, ctypes.byref(desc),
        _ptr(q_packed, "q_packed", dt, shp), _ptr(k_packed, "k_packed", dt, shp),
        _ptr(kv_idx, "kv_idx", torch.int32, (desc.B, desc.H, p.num_q_tiles, p.max_kept)),
        _ptr(kv_cnt, "kv_cnt", torch.int32, (desc.B, desc.H, p.num_q_tiles)),
        _ptr(tile_scores, "tile_scores", torch.float32, (desc.B, desc.H, p.num_tiles, p.num_tiles), optional=True),
        _ptr(workspace, "workspace", torch.uint8), ctypes.c_size_t(workspace.numel()),
        _stream(stream, dev))
    return kv_idx, kv_cnt, workspace


def ssta_attention_fwd(desc: Desc, q_packed, k_packed, v_packed, kv_idx, kv_cnt, o_packed=None, lse=None,
                       workspace=None, stream=None):
    """Step 4 (block-sparse attention): returns (o_packed [B,H,Lq,D], lse [B,H,Lq] fp32, workspace)."""
    p = ssta_plan(desc)
    dt = _torch_dtype(desc)
    dev = q_packed.device
    shp = (desc.B, desc.H, p.packed_len, desc.D)
    if o_packed is None:
        o_packed = torch.empty(shp, dtype=dt, device=dev)
    if lse is None:
        lse = torch.empty((desc.B, desc.H, p.packed_len), dtype=torch.float32, device=dev)
    if workspace is None:
        workspace = _workspace(p.attn_workspace_bytes, dev)
    _call(
        "ssta_attention_fwd", dev, ctypes.byref(desc),
        _ptr(q_packed, "q_packed", dt, shp), _ptr(k_packed, "k_packed", dt, shp),
        _ptr(v_packed, "v_packed", dt, shp),
        _ptr(kv_idx, "kv_idx", torch.int32, (desc.B, desc.H, p.num_q_tiles, p.max_kept)),
        _ptr(kv_cnt, "kv_cnt", torch.int32, (desc.B, desc.H, p.num_q_tiles)),
        _ptr(o_packed, "o_packed", dt, shp), _ptr(lse, "lse", torch.float32, shp[:3]),
        _ptr(workspace, "workspace", torch.uint8), ctypes.c_size_t(workspace.numel()),
        _stream(stream, dev))
    return o_packed, lse, workspace


def ssta_attention_bwd(desc: Desc, q_packed, k_packed, v_packed, o_packed, lse, do_packed, kv_idx, kv_cnt,
                       dq=None, dk=None, dv=None, workspace=None, stream=None):
    """Backward of Step 4: returns (dq, dk, dv [B,H,Lq,D], workspace)."""
    p = ssta_plan(desc)
    dt = _torch_dtype(desc)
    dev = q_packed.device
    shp = (desc.B, desc.H, p.packed_len, desc.D)
    dq = torch.empty(shp, dtype=dt, device=dev) if dq is None else dq
    dk = torch.empty(shp, dtype=dt, device=dev) if dk is None else dk
    dv = torch.empty(shp, dtype=dt, device=dev) if dv is None else dv
    if workspace is None:
        workspace = _workspace(p.bwd_workspace_bytes, dev)
    _call(
        "ssta_attention_bwd", dev, ctypes.byref(desc),
        _ptr(q_packed, "q_packed", dt, shp), _ptr(k_packed, "k_packed", dt, shp), _ptr(v_packed, "v_packed", dt, shp),
        _ptr(o_packed, "o_packed", dt, shp), _ptr(lse, "lse", torch.float32, shp[:3]),
        _ptr(do_packed, "do_packed", dt, shp),
        _ptr(kv_idx, "kv_idx", torch.int32, (desc.B, desc.H, p.num_q_tiles, p.max_kept)),
        _ptr(kv_cnt, "kv_cnt", torch.int32, (desc.B, desc.H, p.num_q_tiles)),
        _ptr(dq, "dq", dt, shp), _ptr(dk, "dk", dt, shp), _ptr(dv, "dv", dt, shp),
        _ptr(workspace, "workspace", torch.uint8), ctypes.c_size_t(workspace.numel()),
        _stream(stream, dev))
    return dq, dk, dv, workspace


def ssta_tile_unorder(desc: Desc, x_packed, x_raster=None, x_text=None, stream=None, want_text=True):
    """Inverse of Step 1: packed -> (raster [B,H,T,Y,X,D], text [B,H,L,D] or None)."""
    p = ssta_plan(desc)
    dt = _torch_dtype(desc)
    dev = x_packed.device
    if x_raster is None:
        x_raster = torch.empty((desc.B, desc.H, desc.T, desc.Y, desc.X, desc.D), dtype=dt, device=dev)
    if x_text is None and want_text and desc.L_text > 0:
        x_text = torch.empty((desc.B, desc.H, desc.L_text, desc.D), dtype=dt, device=dev)
    _call(
        "ssta_tile_unorder", dev, ctypes.byref(desc),
        _ptr(x_packed, "x_packed", dt, (desc.B, desc.H, p.packed_len, desc.D)),
        _ptr(x_raster, "x_raster", dt, (desc.B, desc.H, desc.T, desc.Y, desc.X, desc.D)),
        _ptr(x_text, "x_text", dt, (desc.B, desc.H, desc.L_text, desc.D), optional=True),
        _stream(stream, dev))
    return x_raster, x_text


def ssta_read_device_status(workspace, stream=None) -> int:
    """Device status word of a workspace (0 = no device-side error).  Synchronises the stream."""
    code = ctypes.c_int32(-1)
    _call("ssta_read_device_status", workspace.device, _ptr(workspace, "workspace", torch.uint8),
          _stream(stream, workspace.device), ctypes.byref(code))
    return int(code.value)


def ssta_forward(desc: Desc, q, k, v, q_text=None, k_text=None, v_text=None, stream=None, tile_scores=None):
    """The whole SSTA forward: reorder q, k, v; build the block mask; attend; unorder O.

    Returns a dict with O (raster), O_text, and the intermediate packed tensors,
    lists, LSE and workspaces.
    """
    qp = ssta_tile_reorder(desc, q, q_text, stream=stream)
    kp = ssta_tile_reorder(desc, k, k_text, stream=stream)
    vp = ssta_tile_reorder(desc, v, v_text, stream=stream)
    kv_idx, kv_cnt, ws_mask = ssta_build_block_mask(desc, qp, kp, tile_scores=tile_scores, stream=stream)
    op, lse, ws_attn = ssta_attention_fwd(desc, qp, kp, vp, kv_idx, kv_cnt, stream=stream)
    o, o_text = ssta_tile_unorder(desc, op, stream=stream)
    return dict(O=o, O_text=o_text, qp=qp, kp=kp, vp=vp, kv_idx=kv_idx, kv_cnt=kv_cnt, O_packed=op, LSE=lse,
                ws_mask=ws_mask, ws_attn=ws_attn)
