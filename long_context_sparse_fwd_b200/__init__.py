"""Python binding of the sm_100a CSA / HCA attention library (libcsa.so, C ABI in include/csa.h).

Argument marshalling only: every step of the forward runs in the library's CUDA kernels. PyTorch
provides device memory and the current stream. There is no CPU path: if the library is missing
or the tensors are not on a CUDA device the calls raise.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional, Tuple

import torch

__all__ = [
    "CSAError", "lib", "library_path", "compress", "index_topk", "attend", "hca_attend", "csa_forward",
    "hca_forward", "decode", "hca_decode", "swa_attend", "compress_append", "out_proj", "workspace_size",
    "quantize_mxfp4", "decode_fp4", "index_topk_fp4",
    "get_device_status", "OP",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libcsa.so")
_lib = None

OP = {"index_topk": 1, "attend": 2, "csa_forward": 3, "hca_forward": 4, "decode": 5, "hca_decode": 6,
      "out_proj": 7}
_STATUS = {0: "CSA_OK", 1: "CSA_ERR_INVALID_ARG", 2: "CSA_ERR_UNSUPPORTED", 3: "CSA_ERR_CUDA",
           4: "CSA_ERR_TIMEOUT", 5: "CSA_ERR_WORKSPACE"}


class CSAError(RuntimeError):
    def __init__(self, call: str, code: int):
        super().__init__(f"{call} failed: {_STATUS.get(code, code)}")
        self.code = code


class _Dims(ctypes.Structure):
    _fields_ = [("S", ctypes.c_int64), ("T", ctypes.c_int64), ("B", ctypes.c_int32), ("H", ctypes.c_int32),
                ("D", ctypes.c_int32), ("HI", ctypes.c_int32), ("dI", ctypes.c_int32), ("k", ctypes.c_int32),
                ("W", ctypes.c_int32)]


def library_path() -> str:
    return _LIB_PATH


def lib():
    """Load libcsa.so (built by ``build.build()``); raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(f"CUDA library not built: {_LIB_PATH} is missing (run __graft_entry__.build())")
        L = ctypes.CDLL(_LIB_PATH)
        P, I64, I32, F64, F32, SZ = (ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_double,
                                     ctypes.c_float, ctypes.c_size_t)
        sig = {
            "csa_status_str": (ctypes.c_char_p, [I32]),
            "csa_version": (ctypes.c_char_p, []),
            "csa_workspace_size": (SZ, [I32, ctypes.POINTER(_Dims)]),
            "csa_get_device_status": (I32, [P, ctypes.POINTER(ctypes.c_int32), P]),
            "csa_compress": (I32, [P, P, P, I64, I64, I32, I32, I32, I32, F64, F64, P, P, P]),
            "csa_index_topk": (I32, [P, P, P, I64, I64, I64, I32, I32, I32, I32, P, P, SZ, P]),
            "csa_attend": (I32, [P, P, P, P, P, I64, I64, I32, I32, I64, I32, I32, I32, I32, F64, F64, F32, P, P,
                                 SZ, P]),
            "hca_attend": (I32, [P, P, P, P, I64, I64, I32, I32, I64, I32, I32, I32, F64, F64, F32, P, P, SZ, P]),
            "csa_forward": (I32, [P, P, P, P, P, P, P, P, I64, I64, I32, I32, I32, I32, I32, I32, I32, I32, I32,
                                  F64, F64, F32, P, P, P, P, P, SZ, P]),
            "hca_forward": (I32, [P, P, P, P, P, I64, I64, I32, I32, I32, I32, I32, I32, F64, F64, F32, P, P, P, P,
                                  SZ, P]),
            "csa_decode": (I32, [P, P, P, P, P, P, P, P, P, P, I32, I32, I32, I64, I32, I32, I32, I32, I32, I64,
                                 F64, F64, F32, P, P, P, SZ, P]),
            "hca_decode": (I32, [P, P, P, P, P, P, P, I32, I32, I32, I64, I32, I32, I64, F64, F64, F32, P, P, SZ, P]),
            "swa_attend": (I32, [P, P, P, I64, I64, I32, I32, I32, I32, F64, F32, P, P, SZ, P]),
            "csa_compress_append": (I32, [P, P, P, P, P, I32, I32, I32, I32, I32, I64, F64, F64, P, P, P, P, I64, P,
                                          I32, P]),
            "csa_out_proj": (I32, [P, P, P, I64, I32, I32, I32, I32, I32, P, P, P, SZ, P]),
            "csa_quantize_mxfp4": (I32, [P, I64, I32, P, P, P]),
            "csa_index_topk_fp4": (I32, [P, P, P, P, P, I64, I64, I64, I32, I32, I32, I32, P, P, SZ, P]),
            "csa_decode_fp4": (I32, [P, P, P, P, P, P, P, P, P, P, P, P, I32, I32, I32, I64, I32, I32, I32, I32, I32,
                                     I64, F64, F64, F32, P, P, P, SZ, P]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


# ---- marshalling ----------------------------------------------------------------------------------

def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _dev(t: Optional[torch.Tensor], dtype, name: str, shape=None):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    return t


def _stream(stream: Optional[torch.cuda.Stream]):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check(call: str, code: int):
    if code != 0:
        raise CSAError(call, code)


def workspace_size(op: str, S=0, T=0, B=0, H=0, D=0, HI=0, dI=0, k=0, W=0) -> int:
    d = _Dims(S, T, B, H, D, HI, dI, k, W)
    return int(lib().csa_workspace_size(OP[op], ctypes.byref(d)))


def _workspace(op: str, device, ws: Optional[torch.Tensor], **dims) -> torch.Tensor:
    # the library checks the size it is given (decode accepts less than the recommended size)
    if ws is None:
        ws = torch.empty(workspace_size(op, **dims), dtype=torch.uint8, device=device)
    return ws


def get_device_status(ws: torch.Tensor, stream=None) -> int:
    v = ctypes.c_int32(0)
    _check("csa_get_device_status", lib().csa_get_device_status(_ptr(ws), ctypes.byref(v), _stream(stream)))
    return int(v.value)


# ---- the calls ----------------------------------------------------------------------------------------

def compress(kv, gate, pos_bias, m: int, L: int, rope_dim: int, theta_cmp: float, theta_tok: float,
             C=None, kv_rot=None, want_kv_rot: bool = True, pos0: int = 0,
             stream=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """kv, gate [N, D] by position (N = pos0 + S). Writes the entries closing in the chunk
    [pos0, N) into C [N // m, D] and rows [pos0, N) into kv_rot [N, D]; with pos0 > 0 pass the
    caches (C, kv_rot) holding the earlier chunks."""
    N, D = kv.shape
    S = N - int(pos0)
    if S < 0:
        raise ValueError("kv holds fewer rows than pos0")
    T = N // m
    _dev(kv, torch.bfloat16, "kv", (N, D))
    _dev(gate, torch.bfloat16, "gate", (N, D))
    _dev(pos_bias, torch.float32, "pos_bias", (L,))
    if pos0 > 0 and (C is None or (want_kv_rot and kv_rot is None)):
        raise ValueError("a chunk at pos0 > 0 needs the caches C and kv_rot of the earlier chunks")
    C = torch.empty(T, D, dtype=torch.bfloat16, device=kv.device) if C is None else _dev(C, torch.bfloat16, "C", (T, D))
    if want_kv_rot:
        kv_rot = torch.empty_like(kv) if kv_rot is None else _dev(kv_rot, torch.bfloat16, "kv_rot", (N, D))
    else:
        kv_rot = None
    _check("csa_compress", lib().csa_compress(_ptr(kv), _ptr(gate), _ptr(pos_bias), S, int(pos0), D, m, L, rope_dim,
                                              float(theta_cmp), float(theta_tok), _ptr(C), _ptr(kv_rot),
                                              _stream(stream)))
    return C, kv_rot


def index_topk(qI, kI, w, m: int, k: int, idx=None, workspace=None, pos0: int = 0, stream=None) -> torch.Tensor:
    """qI [S, HI, dI], w [S, HI] of the queries at positions pos0 .. pos0+S-1; kI [T, dI] every entry
    so far. Returns idx [S, k]."""
    S, HI, dI = qI.shape
    T = kI.shape[0]
    _dev(qI, torch.bfloat16, "qI")
    _dev(kI, torch.bfloat16, "kI", (T, dI))
    _dev(w, torch.float32, "w", (S, HI))
    idx = torch.empty(S, k, dtype=torch.int32, device=qI.device) if idx is None else _dev(idx, torch.int32, "idx", (S, k))
    ws = _workspace("index_topk", qI.device, workspace, S=S, T=T, HI=HI, dI=dI, k=k)
    _check("csa_index_topk", lib().csa_index_topk(_ptr(qI), _ptr(kI), _ptr(w), S, int(pos0), T, HI, dI, m, k,
                                                  _ptr(idx), _ptr(ws), ws.numel(), _stream(stream)))
    return idx


def attend(q, C, kv_rot, idx, sinks, m: int, W: int, rope_dim: int, theta_tok: float, theta_cmp: float,
           softmax_scale: float = 0.0, o=None, workspace=None, pos0: int = 0, stream=None) -> torch.Tensor:
    """q [S, H, D] and idx [S, k] of the queries at positions pos0 .. pos0+S-1; C [T, D]; kv_rot
    [pos0 + S, D] by position. Returns o [S, H, D] fp32."""
    S, H, D = q.shape
    T = C.shape[0]
    k = idx.shape[1]
    _dev(q, torch.bfloat16, "q")
    _dev(C, torch.bfloat16, "C", (T, D))
    _dev(kv_rot, torch.bfloat16, "kv_rot", (int(pos0) + S, D))
    _dev(idx, torch.int32, "idx", (S, k))
    _dev(sinks, torch.float32, "sinks", (H,))
    o = torch.empty(S, H, D, dtype=torch.float32, device=q.device) if o is None else _dev(o, torch.float32, "o", (S, H, D))
    ws = _workspace("attend", q.device, workspace)
    _check("csa_attend", lib().csa_attend(_ptr(q), _ptr(C), _ptr(kv_rot), _ptr(idx), _ptr(sinks), S, int(pos0), H, D,
                                          T, k, W, rope_dim, m, float(theta_tok), float(theta_cmp),
                                          float(softmax_scale), _ptr(o), _ptr(ws), ws.numel(), _stream(stream)))
    return o


def hca_attend(q, C, kv_rot, sinks, m: int, W: int, rope_dim: int, theta_tok: float, theta_cmp: float,
               softmax_scale: float = 0.0, o=None, workspace=None, pos0: int = 0, stream=None) -> torch.Tensor:
    S, H, D = q.shape
    T = C.shape[0]
    _dev(q, torch.bfloat16, "q")
    _dev(C, torch.bfloat16, "C", (T, D))
    _dev(kv_rot, torch.bfloat16, "kv_rot", (int(pos0) + S, D))
    _dev(sinks, torch.float32, "sinks", (H,))
    o = torch.empty(S, H, D, dtype=torch.float32, device=q.device) if o is None else _dev(o, torch.float32, "o", (S, H, D))
    ws = _workspace("attend", q.device, workspace)
    _check("hca_attend", lib().hca_attend(_ptr(q), _ptr(C), _ptr(kv_rot), _ptr(sinks), S, int(pos0), H, D, T, W,
                                          rope_dim, m, float(theta_tok), float(theta_cmp), float(softmax_scale),
                                          _ptr(o), _ptr(ws), ws.numel(), _stream(stream)))
    return o


def csa_forward(q, kv, gate, pos_bias, qI, kI, w, sinks, m: int, L: int, k: int, W: int, rope_dim: int,
                theta_tok: float, theta_cmp: float, softmax_scale: float = 0.0, out=None, workspace=None,
                pos0: int = 0, stream=None):
    """Returns (o, C, kv_rot, idx). `out` may pass preallocated (o, C, kv_rot, idx). For a chunk at
    pos0 > 0, kv and gate are [pos0 + S, D] by position, kI [(pos0 + S) // m, dI] holds every entry's
    index key, and `out` must carry the caches C [(pos0 + S) // m, D] and kv_rot [pos0 + S, D] of the
    earlier chunks; q, qI, w, o and idx hold the chunk's S rows."""
    S, H, D = q.shape
    HI, dI = qI.shape[1], qI.shape[2]
    N = int(pos0) + S
    T = N // m
    for t, n, dt, shp in ((q, "q", torch.bfloat16, None), (kv, "kv", torch.bfloat16, (N, D)),
                          (gate, "gate", torch.bfloat16, (N, D)), (pos_bias, "pos_bias", torch.float32, None),
                          (qI, "qI", torch.bfloat16, (S, HI, dI)), (kI, "kI", torch.bfloat16, (T, dI)),
                          (w, "w", torch.float32, (S, HI)), (sinks, "sinks", torch.float32, None)):
        _dev(t, dt, n, shp)
    if out is None:
        if pos0 > 0:
            raise ValueError("a chunk at pos0 > 0 needs out=(o, C, kv_rot, idx) with the earlier chunks' caches")
        dev = q.device
        out = (torch.empty(S, H, D, dtype=torch.float32, device=dev), torch.empty(T, D, dtype=torch.bfloat16, device=dev),
               torch.empty(N, D, dtype=torch.bfloat16, device=dev), torch.empty(S, k, dtype=torch.int32, device=dev))
    o, C, kv_rot, idx = out
    _dev(o, torch.float32, "o", (S, H, D))
    _dev(C, torch.bfloat16, "C", (T, D))
    _dev(kv_rot, torch.bfloat16, "kv_rot", (N, D))
    _dev(idx, torch.int32, "idx", (S, k))
    ws = _workspace("csa_forward", q.device, workspace, S=S, T=T, HI=HI, dI=dI, k=k)
    _check("csa_forward", lib().csa_forward(_ptr(q), _ptr(kv), _ptr(gate), _ptr(pos_bias), _ptr(qI), _ptr(kI), _ptr(w),
                                            _ptr(sinks), S, int(pos0), H, D, HI, dI, m, L, k, W, rope_dim,
                                            float(theta_tok), float(theta_cmp), float(softmax_scale), _ptr(C),
                                            _ptr(kv_rot), _ptr(idx), _ptr(o), _ptr(ws), ws.numel(), _stream(stream)))
    return o, C, kv_rot, idx


def hca_forward(q, kv, gate, pos_bias, sinks, m: int, L: int, W: int, rope_dim: int, theta_tok: float,
                theta_cmp: float, softmax_scale: float = 0.0, out=None, workspace=None, pos0: int = 0, stream=None):
    """Returns (o, C, kv_rot). For a chunk at pos0 > 0 see csa_forward (out = (o, C, kv_rot))."""
    S, H, D = q.shape
    N = int(pos0) + S
    T = N // m
    for t, n, dt, shp in ((q, "q", torch.bfloat16, None), (kv, "kv", torch.bfloat16, (N, D)),
                          (gate, "gate", torch.bfloat16, (N, D)), (pos_bias, "pos_bias", torch.float32, None),
                          (sinks, "sinks", torch.float32, None)):
        _dev(t, dt, n, shp)
    if out is None:
        if pos0 > 0:
            raise ValueError("a chunk at pos0 > 0 needs out=(o, C, kv_rot) with the earlier chunks' caches")
        dev = q.device
        out = (torch.empty(S, H, D, dtype=torch.float32, device=dev), torch.empty(T, D, dtype=torch.bfloat16, device=dev),
               torch.empty(N, D, dtype=torch.bfloat16, device=dev))
    o, C, kv_rot = out
    _dev(o, torch.float32, "o", (S, H, D))
    _dev(C, torch.bfloat16, "C", (T, D))
    _dev(kv_rot, torch.bfloat16, "kv_rot", (N, D))
    ws = _workspace("hca_forward", q.device, workspace)
    _check("hca_forward", lib().hca_forward(_ptr(q), _ptr(kv), _ptr(gate), _ptr(pos_bias), _ptr(sinks), S, int(pos0),
                                            H, D, m, L, W, rope_dim, float(theta_tok), float(theta_cmp),
                                            float(softmax_scale), _ptr(C), _ptr(kv_rot), _ptr(o), _ptr(ws),
                                            ws.numel(), _stream(stream)))
    return o, C, kv_rot


def decode(q, qI, w, kI, win, sinks, P: int, k: int, rope_dim: int, theta_tok: float, theta_cmp: float,
           C=None, c8=None, c8_scale=None, c_rope=None, softmax_scale: float = 0.0, o=None, idx=None,
           workspace=None, stream=None):
    """Returns (o [B,H,D] fp32, idx [B,k] int32)."""
    B, H, D = q.shape
    HI, dI = qI.shape[1], qI.shape[2]
    T = kI.shape[1]
    W = win.shape[1]
    _dev(q, torch.bfloat16, "q")
    _dev(qI, torch.bfloat16, "qI")
    _dev(w, torch.float32, "w", (B, HI))
    _dev(kI, torch.bfloat16, "kI", (B, T, dI))
    _dev(win, torch.bfloat16, "win", (B, W, D))
    _dev(sinks, torch.float32, "sinks", (H,))
    if C is not None:
        _dev(C, torch.bfloat16, "C", (B, T, D))
    else:
        _dev(c8, torch.uint8, "c8", (B, T, D - rope_dim))
        _dev(c8_scale, torch.float32, "c8_scale", (B, T))
        _dev(c_rope, torch.bfloat16, "c_rope", (B, T, rope_dim))
    o = torch.empty(B, H, D, dtype=torch.float32, device=q.device) if o is None else _dev(o, torch.float32, "o", (B, H, D))
    idx = torch.empty(B, k, dtype=torch.int32, device=q.device) if idx is None else _dev(idx, torch.int32, "idx", (B, k))
    ws = _workspace("decode", q.device, workspace, B=B, T=T, k=k)
    _check("csa_decode", lib().csa_decode(_ptr(q), _ptr(qI), _ptr(w), _ptr(kI), _ptr(C), _ptr(c8), _ptr(c8_scale),
                                          _ptr(c_rope), _ptr(win), _ptr(sinks), B, H, D, T, HI, dI, k, W, rope_dim,
                                          int(P), float(theta_tok), float(theta_cmp), float(softmax_scale), _ptr(idx),
                                          _ptr(o), _ptr(ws), ws.numel(), _stream(stream)))
    return o, idx


def quantize_mxfp4(x, codes=None, scales=None, stream=None):
    """MXFP4 (OCP Microscaling) of bf16 rows x [..., d] (d a multiple of 32): returns
    (codes [..., d/2] uint8, two E2M1 codes per byte with channel 2i in the low nibble,
    scales [..., d/32] uint8 E8M0)."""
    _dev(x, torch.bfloat16, "x")
    d = x.shape[-1]
    rows = x.numel() // d if d else 0
    shape = tuple(x.shape[:-1])
    codes = torch.empty(shape + (d // 2,), dtype=torch.uint8, device=x.device) if codes is None else \
        _dev(codes, torch.uint8, "codes", shape + (d // 2,))
    scales = torch.empty(shape + (d // 32,), dtype=torch.uint8, device=x.device) if scales is None else \
        _dev(scales, torch.uint8, "scales", shape + (d // 32,))
    _check("csa_quantize_mxfp4", lib().csa_quantize_mxfp4(_ptr(x), rows, d, _ptr(codes), _ptr(scales), _stream(stream)))
    return codes, scales


def index_topk_fp4(qc, qs, w, kc, ks, m: int, k: int, idx=None, workspace=None, pos0: int = 0,
                   stream=None) -> torch.Tensor:
    """Prefill lightning indexer + top-k on MXFP4 operands (csa_quantize_mxfp4 layout): qc [S, HI, dI/2],
    qs [S, HI, dI/32], kc [T, dI/2], ks [T, dI/32] uint8; w [S, HI] fp32. Returns idx [S, k] int32."""
    S, HI, half = qc.shape
    dI = 2 * half
    T = kc.shape[0]
    _dev(qc, torch.uint8, "qI codes")
    _dev(qs, torch.uint8, "qI scales", (S, HI, dI // 32))
    _dev(kc, torch.uint8, "kI codes", (T, dI // 2))
    _dev(ks, torch.uint8, "kI scales", (T, dI // 32))
    _dev(w, torch.float32, "w", (S, HI))
    idx = torch.empty(S, k, dtype=torch.int32, device=qc.device) if idx is None else _dev(idx, torch.int32, "idx", (S, k))
    ws = _workspace("attend", qc.device, workspace)
    _check("csa_index_topk_fp4", lib().csa_index_topk_fp4(_ptr(qc), _ptr(qs), _ptr(w), _ptr(kc), _ptr(ks), S, int(pos0),
                                                          T, HI, dI, m, k, _ptr(idx), _ptr(ws), ws.numel(),
                                                          _stream(stream)))
    return idx


def decode_fp4(q, qI_codes, qI_scales, w, kI_codes, kI_scales, win, sinks, P: int, k: int, rope_dim: int,
               theta_tok: float, theta_cmp: float, C=None, c8=None, c8_scale=None, c_rope=None,
               softmax_scale: float = 0.0, o=None, idx=None, workspace=None, stream=None):
    """csa_decode with the indexer's q^I and k^I in MXFP4 (codes and scales as quantize_mxfp4 returns
    them: qI [B,HI,dI/2] + [B,HI,dI/32], kI [B,T,dI/2] + [B,T,dI/32]). Returns (o [B,H,D] fp32,
    idx [B,k] int32)."""
    B, H, D = q.shape
    HI, dI = qI_codes.shape[1], 2 * qI_codes.shape[2]
    T = kI_codes.shape[1]
    W = win.shape[1]
    _dev(q, torch.bfloat16, "q")
    _dev(qI_codes, torch.uint8, "qI_codes", (B, HI, dI // 2))
    _dev(qI_scales, torch.uint8, "qI_scales", (B, HI, dI // 32))
    _dev(w, torch.float32, "w", (B, HI))
    _dev(kI_codes, torch.uint8, "kI_codes", (B, T, dI // 2))
    _dev(kI_scales, torch.uint8, "kI_scales", (B, T, dI // 32))
    _dev(win, torch.bfloat16, "win", (B, W, D))
    _dev(sinks, torch.float32, "sinks", (H,))
    if C is not None:
        _dev(C, torch.bfloat16, "C", (B, T, D))
    else:
        _dev(c8, torch.uint8, "c8", (B, T, D - rope_dim))
        _dev(c8_scale, torch.float32, "c8_scale", (B, T))
        _dev(c_rope, torch.bfloat16, "c_rope", (B, T, rope_dim))
    o = torch.empty(B, H, D, dtype=torch.float32, device=q.device) if o is None else _dev(o, torch.float32, "o", (B, H, D))
    idx = torch.empty(B, k, dtype=torch.int32, device=q.device) if idx is None else _dev(idx, torch.int32, "idx", (B, k))
    ws = _workspace("decode", q.device, workspace, B=B, T=T, k=k)
    _check("csa_decode_fp4", lib().csa_decode_fp4(
        _ptr(q), _ptr(qI_codes), _ptr(qI_scales), _ptr(w), _ptr(kI_codes), _ptr(kI_scales), _ptr(C), _ptr(c8),
        _ptr(c8_scale), _ptr(c_rope), _ptr(win), _ptr(sinks), B, H, D, T, HI, dI, k, W, rope_dim, int(P),
        float(theta_tok), float(theta_cmp), float(softmax_scale), _ptr(idx), _ptr(o), _ptr(ws), ws.numel(),
        _stream(stream)))
    return o, idx


def hca_decode(q, win, sinks, P: int, rope_dim: int, theta_tok: float, theta_cmp: float, C=None, c8=None,
               c8_scale=None, c_rope=None, T: Optional[int] = None, softmax_scale: float = 0.0, o=None,
               workspace=None, stream=None) -> torch.Tensor:
    """HCA decode: every cached entry (bf16 C [B,T,D], or the FP8 triplet) plus the window rows
    win [B,W,D] and the sink. With no entry cache (T = 0) it is the sliding-window-only decode.
    Returns o [B,H,D] fp32."""
    B, H, D = q.shape
    W = win.shape[1]
    _dev(q, torch.bfloat16, "q")
    _dev(win, torch.bfloat16, "win", (B, W, D))
    _dev(sinks, torch.float32, "sinks", (H,))
    if C is not None:
        T = C.shape[1]
        _dev(C, torch.bfloat16, "C", (B, T, D))
    elif c8 is not None:
        T = c8.shape[1]
        _dev(c8, torch.uint8, "c8", (B, T, D - rope_dim))
        _dev(c8_scale, torch.float32, "c8_scale", (B, T))
        _dev(c_rope, torch.bfloat16, "c_rope", (B, T, rope_dim))
    else:
        T = 0
    o = torch.empty(B, H, D, dtype=torch.float32, device=q.device) if o is None else _dev(o, torch.float32, "o", (B, H, D))
    ws = _workspace("hca_decode", q.device, workspace, B=B, T=T, W=W)
    _check("hca_decode", lib().hca_decode(_ptr(q), _ptr(C), _ptr(c8), _ptr(c8_scale), _ptr(c_rope), _ptr(win),
                                          _ptr(sinks), B, H, D, T, W, rope_dim, int(P), float(theta_tok),
                                          float(theta_cmp), float(softmax_scale), _ptr(o), _ptr(ws), ws.numel(),
                                          _stream(stream)))
    return o


def swa_attend(q, kv_rot, sinks, W: int, rope_dim: int, theta_tok: float, softmax_scale: float = 0.0, o=None,
               workspace=None, pos0: int = 0, stream=None) -> torch.Tensor:
    """Sliding-window-only layer prefill of the queries at positions pos0 .. pos0+S-1: window rows
    kv_rot [pos0 + S, D] by position and the sink. Returns o [S,H,D] fp32."""
    S, H, D = q.shape
    _dev(q, torch.bfloat16, "q")
    _dev(kv_rot, torch.bfloat16, "kv_rot", (int(pos0) + S, D))
    _dev(sinks, torch.float32, "sinks", (H,))
    o = torch.empty(S, H, D, dtype=torch.float32, device=q.device) if o is None else _dev(o, torch.float32, "o", (S, H, D))
    ws = _workspace("attend", q.device, workspace)
    _check("swa_attend", lib().swa_attend(_ptr(q), _ptr(kv_rot), _ptr(sinks), S, int(pos0), H, D, W, rope_dim,
                                          float(theta_tok), float(softmax_scale), _ptr(o), _ptr(ws), ws.numel(),
                                          _stream(stream)))
    return o


def compress_append(x_new, g_new, pos_bias, state_x, state_g, P: int, m: int, rope_dim: int, theta_cmp: float,
                    theta_tok: float, C=None, c8=None, c8_scale=None, c_rope=None, win=None, stream=None) -> None:
    """The compressor's decode step for the token at position P (the same for every sequence): writes
    it into the state rings [B,L,D], emits entry (P+1)/m - 1 into the bf16 cache C [B,Tcap,D] (or the
    FP8 triplet) when (P+1) % m == 0, and writes its rotated window row into win [B,W,D] at slot
    (W-1-P) mod W."""
    B, D = x_new.shape
    L = state_x.shape[1]
    _dev(x_new, torch.bfloat16, "x_new")
    _dev(g_new, torch.bfloat16, "g_new", (B, D))
    _dev(pos_bias, torch.float32, "pos_bias", (L,))
    _dev(state_x, torch.bfloat16, "state_x", (B, L, D))
    _dev(state_g, torch.bfloat16, "state_g", (B, L, D))
    if C is not None:
        Tcap = C.shape[1]
        _dev(C, torch.bfloat16, "C", (B, Tcap, D))
    else:
        Tcap = c8.shape[1]
        _dev(c8, torch.uint8, "c8", (B, Tcap, D - rope_dim))
        _dev(c8_scale, torch.float32, "c8_scale", (B, Tcap))
        if rope_dim > 0:
            _dev(c_rope, torch.bfloat16, "c_rope", (B, Tcap, rope_dim))
    W = 0
    if win is not None:
        W = win.shape[1]
        _dev(win, torch.bfloat16, "win", (B, W, D))
    _check("csa_compress_append", lib().csa_compress_append(
        _ptr(x_new), _ptr(g_new), _ptr(pos_bias), _ptr(state_x), _ptr(state_g), B, D, m, L, rope_dim, int(P),
        float(theta_cmp), float(theta_tok), _ptr(C), _ptr(c8), _ptr(c8_scale), _ptr(c_rope), Tcap, _ptr(win), W,
        _stream(stream)))


def out_proj(o, wa, wb, z=None, out=None, workspace=None, stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Grouped low-rank output projection: o [S,H,D] (or [S,H*D]) bf16, wa [G,R,(H/G)*D] bf16,
    wb [hidden,G*R] bf16. Returns (z [S,G*R] bf16, out [S,hidden] bf16)."""
    S = o.shape[0]
    G, R, K = wa.shape
    hidden = wb.shape[0]
    if o.dim() == 3:
        H, D = o.shape[1], o.shape[2]
    else:   # [S, H*D]: only the per-group width K and the row length matter
        H, D = G, o.shape[1] // G
    HD = H * D
    _dev(o, torch.bfloat16, "o")
    _dev(wa, torch.bfloat16, "wa", (G, R, K))
    _dev(wb, torch.bfloat16, "wb", (hidden, G * R))
    if HD != G * K:
        raise ValueError(f"o has {HD} channels per token; wa expects {G} groups of {K}")
    z = torch.empty(S, G * R, dtype=torch.bfloat16, device=o.device) if z is None else _dev(z, torch.bfloat16, "z", (S, G * R))
    out = torch.empty(S, hidden, dtype=torch.bfloat16, device=o.device) if out is None else \
        _dev(out, torch.bfloat16, "out", (S, hidden))
    ws = _workspace("out_proj", o.device, workspace)
    _check("csa_out_proj", lib().csa_out_proj(_ptr(o), _ptr(wa), _ptr(wb), S, H, D, G, R, hidden, _ptr(z), _ptr(out),
                                              _ptr(ws), ws.numel(), _stream(stream)))
    return z, out
