"""fp64 CPU oracle of the CSA / HCA attention forward (test infrastructure only).

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg may import this
package. The product path (the CUDA library and its binding) never does, and the oracle never
imports the product path.

The arithmetic lives in ``csa_oracle.c`` (plain C, double precision, OpenMP over query rows);
this module compiles it with gcc and marshals numpy arrays into it. The grouped output projection
(``out_proj``) is two fp64 matrix products, done with numpy's. bf16 arrays are passed as
their raw uint16 bit patterns, FP8 E4M3 caches as raw bytes, so the oracle reads exactly the
values the GPU reads.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "csa_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libcsa_oracle.so")
_lib = None

_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_I32 = ctypes.c_int
_F64 = ctypes.c_double


def build(force: bool = False) -> str:
    """Compile the oracle (gcc -O2, IEEE semantics: no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fPIC", "-shared", "-std=c99",
               "-Wall", "-o", _LIB_PATH + ".tmp", _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(_LIB_PATH + ".tmp", _LIB_PATH)
    return _LIB_PATH


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB_PATH)
        L.orc_bf16_to_f64.restype = _F64
        L.orc_bf16_to_f64.argtypes = [ctypes.c_uint16]
        L.orc_e4m3_to_f64.restype = _F64
        L.orc_e4m3_to_f64.argtypes = [ctypes.c_uint8]
        L.orc_e4m3_from_f32.restype = ctypes.c_uint8
        L.orc_e4m3_from_f32.argtypes = [ctypes.c_float]
        L.orc_e4m3_from_f32_array.restype = None
        L.orc_e4m3_from_f32_array.argtypes = [_P, _I64, _P]
        L.orc_fp8_entry_rows.restype = None
        L.orc_fp8_entry_rows.argtypes = [_P, _I64, _I32, _P, _P]
        L.orc_rope.restype = None
        L.orc_rope.argtypes = [_P, _I32, _I32, _F64, _F64]
        L.orc_compress.restype = _I64
        L.orc_compress.argtypes = [_P, _P, _P, _I64, _I32, _I32, _I32, _I32, _F64, _F64, _P, _P]
        L.orc_visible.restype = _I64
        L.orc_visible.argtypes = [_I64, _I32, _I64]
        L.orc_index_scores.restype = None
        L.orc_index_scores.argtypes = [_P, _P, _P, _I64, _I64, _I32, _I32, _I32, _P, _I64, _P]
        L.orc_decode_index_scores.restype = None
        L.orc_decode_index_scores.argtypes = [_P, _P, _P, _I64, _I64, _I32, _I32, _P, _I64, _P]
        L.orc_topk.restype = None
        L.orc_topk.argtypes = [_P, _P, _I64, _I64, _I32, _P]
        L.orc_attend.restype = None
        L.orc_attend.argtypes = [_P, _P, _P, _P, _P, _I64, _I32, _I32, _I64, _I32, _I32, _I32,
                                 _F64, _F64, _I32, _F64, _P, _I64, _P]
        L.orc_decode_attend.restype = None
        L.orc_decode_attend.argtypes = [_P, _P, _P, _P, _P, _P, _P, _P, _I64, _I32, _I32, _I64, _I32,
                                        _I32, _I32, _I64, _F64, _F64, _F64, _P, _I64, _P]
        L.orc_num_threads.restype = _I32
        L.orc_num_threads.argtypes = []
        _lib = L
    return _lib


# ---- marshalling helpers ------------------------------------------------------------------------

def _np(x, dtype=None):
    """numpy view of a CPU tensor / array; bf16 tensors become their uint16 bit patterns."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().cpu().contiguous()
            if x.dtype == torch.bfloat16:
                x = x.view(torch.int16)
                return np.ascontiguousarray(x.numpy().view(np.uint16))
            if x.dtype == torch.float8_e4m3fn:
                x = x.view(torch.uint8)
            x = x.numpy()
    except ImportError:  # pragma: no cover
        pass
    x = np.ascontiguousarray(x)
    if dtype is not None and x.dtype != dtype:
        x = np.ascontiguousarray(x.astype(dtype))
    return x


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def num_threads() -> int:
    return int(lib().orc_num_threads())


def e4m3_encode(x) -> np.ndarray:
    """E4M3 codes (uint8, same shape) of binary32 values: nearest, ties to the even code, finite
    overflow saturating to +-448, NaN -> 0x7F (the OCP FP8 definition's saturating conversion)."""
    x_ = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    out = np.empty(x_.shape, np.uint8)
    lib().orc_e4m3_from_f32_array(_ptr(x_), x_.size, _ptr(out))
    return out


def fp8_entry_rows(x):
    """FP8 form of entry rows x [n, c] (binary32 values of the non-rope channels): per row
    scale = amax / 448 in binary32 (1 for an all-zero row) and codes = E4M3 of x / scale.
    Returns (codes uint8 [n, c], scale float32 [n])."""
    x_ = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    n, c = x_.shape
    codes = np.empty((n, c), np.uint8)
    scale = np.empty(n, np.float32)
    lib().orc_fp8_entry_rows(_ptr(x_), n, c, _ptr(codes), _ptr(scale))
    return codes, scale


def bf16_to_f64(bits: int) -> float:
    return float(lib().orc_bf16_to_f64(int(bits)))


def e4m3_to_f64(code: int) -> float:
    return float(lib().orc_e4m3_to_f64(int(code)))


def rope(x, r: int, pos: float, theta: float) -> np.ndarray:
    """Rotate a copy of x [D] (double) on its last r channels at position pos."""
    v = np.array(x, dtype=np.float64, copy=True)
    lib().orc_rope(_ptr(v), v.shape[-1], int(r), float(pos), float(theta))
    return v


def visible(t: int, m: int, T: int) -> int:
    return int(lib().orc_visible(int(t), int(m), int(T)))


def compress(kv, gate, pos_bias, m: int, L: int, r: int, theta_cmp: float, theta_tok: float,
             want_C: bool = True, want_kv_rot: bool = True):
    """Pooled, rotated entries C [T,D] and rotated raw rows kv_rot [S,D], both float64."""
    kv_, gate_, b_ = _np(kv), _np(gate), _np(pos_bias, np.float32)
    S, D = kv_.shape
    assert b_.shape == (L,)
    T = S // m
    C = np.empty((T, D), np.float64) if want_C else None
    kr = np.empty((S, D), np.float64) if want_kv_rot else None
    got = lib().orc_compress(_ptr(kv_), _ptr(gate_), _ptr(b_), S, D, m, L, r, theta_cmp, theta_tok,
                             _ptr(C), _ptr(kr))
    if got < 0:
        raise ValueError("oracle compress: bad arguments")
    return C, kr


def index_scores(qI, kI, w, m: int, rows=None) -> np.ndarray:
    """I[rows, :T] in float64 (NaN where the entry is not yet visible)."""
    q_, k_, w_ = _np(qI), _np(kI), _np(w, np.float32)
    S, HI, dI = q_.shape
    T = k_.shape[0]
    rows_ = np.arange(S, dtype=np.int64) if rows is None else np.asarray(rows, np.int64)
    out = np.empty((len(rows_), T), np.float64)
    lib().orc_index_scores(_ptr(q_), _ptr(k_), _ptr(w_), S, T, HI, dI, m, _ptr(rows_), len(rows_), _ptr(out))
    return out


def topk(scores, vis, k: int) -> np.ndarray:
    """Top-k per row (ties to the smaller index), ascending order, -1 padded. int32 [n,k]."""
    s_ = np.ascontiguousarray(scores, np.float64)
    v_ = np.ascontiguousarray(vis, np.int64)
    out = np.empty((s_.shape[0], k), np.int32)
    lib().orc_topk(_ptr(s_), _ptr(v_), s_.shape[0], s_.shape[1], int(k), _ptr(out))
    return out


def index_topk(qI, kI, w, m: int, k: int, rows=None):
    """(idx [n,k] int32, scores [n,T] float64) for the listed query rows."""
    S = _np(qI).shape[0]
    T = _np(kI).shape[0]
    rows_ = np.arange(S, dtype=np.int64) if rows is None else np.asarray(rows, np.int64)
    sc = index_scores(qI, kI, w, m, rows_)
    vis = np.array([visible(t, m, T) for t in rows_], np.int64)
    return topk(sc, vis, k), sc


def attend(q, C, kv_rot, idx, sinks, m: int, W: int, r: int, theta_tok: float, theta_cmp: float,
           scale: float = 0.0, rows=None) -> np.ndarray:
    """Attention output [n,H,D] float64 for the listed query rows. idx None = HCA (all visible
    entries). C / kv_rot may be bf16 tensors or float64 arrays (post-RoPE)."""
    q_ = _np(q)
    S, H, D = q_.shape
    C_ = _as_f64(C)
    kr_ = _as_f64(kv_rot)
    T = C_.shape[0]
    idx_ = None if idx is None else _np(idx, np.int32)
    k = 0 if idx_ is None else idx_.shape[1]
    if idx_ is not None:
        assert idx_.shape[0] == S
    s_ = _np(sinks, np.float32)
    rows_ = np.arange(S, dtype=np.int64) if rows is None else np.asarray(rows, np.int64)
    out = np.empty((len(rows_), H, D), np.float64)
    lib().orc_attend(_ptr(q_), _ptr(C_), _ptr(kr_), _ptr(idx_), _ptr(s_), S, H, D, T, k, W, r,
                     theta_tok, theta_cmp, m, scale, _ptr(rows_), len(rows_), _ptr(out))
    return out


def decode_index_topk(qI, w, kI, k: int, rows=None):
    q_, w_, k_ = _np(qI), _np(w, np.float32), _np(kI)
    B, HI, dI = q_.shape
    T = k_.shape[1]
    rows_ = np.arange(B, dtype=np.int64) if rows is None else np.asarray(rows, np.int64)
    sc = np.empty((len(rows_), T), np.float64)
    lib().orc_decode_index_scores(_ptr(q_), _ptr(w_), _ptr(k_), B, T, HI, dI, _ptr(rows_), len(rows_), _ptr(sc))
    vis = np.full(len(rows_), T, np.int64)
    return topk(sc, vis, k), sc


def decode_attend(q, win, idx, sinks, P: int, r: int, theta_tok: float, theta_cmp: float,
                  C=None, c8=None, c8_scale=None, c_rope=None, scale: float = 0.0, rows=None,
                  idx_rows_aligned: bool = False) -> np.ndarray:
    """Decode attention [n,H,D] float64 for sequences rows (default all). idx is [B,k] indexed by
    sequence, or [n,k] aligned with rows when idx_rows_aligned."""
    q_ = _np(q)
    B, H, D = q_.shape
    win_ = _np(win)
    W = win_.shape[1]
    rows_ = np.arange(B, dtype=np.int64) if rows is None else np.asarray(rows, np.int64)
    idx_ = _np(idx, np.int32)
    if idx_rows_aligned:
        full = np.full((B, idx_.shape[1]), -1, np.int32)
        full[rows_] = idx_
        idx_ = full
    k = idx_.shape[1]
    if C is not None:
        C_ = _np(C)
        T = C_.shape[1]
        c8_ = sc_ = cr_ = None
    else:
        C_ = None
        c8_, sc_, cr_ = _np(c8), _np(c8_scale, np.float32), _np(c_rope)
        T = c8_.shape[1]
    s_ = _np(sinks, np.float32)
    out = np.empty((len(rows_), H, D), np.float64)
    lib().orc_decode_attend(_ptr(q_), _ptr(C_), _ptr(c8_), _ptr(sc_), _ptr(cr_), _ptr(win_), _ptr(idx_),
                            _ptr(s_), B, H, D, T, k, W, r, int(P), theta_tok, theta_cmp, scale,
                            _ptr(rows_), len(rows_), _ptr(out))
    return out


def _as_f64(x) -> np.ndarray:
    try:
        import torch
        if isinstance(x, torch.Tensor) and x.dtype == torch.bfloat16:
            return x.detach().cpu().float().double().numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def round_bf16(x) -> np.ndarray:
    """Round float64 values to the nearest bf16 value (8 significant bits, ties to even), as float64.
    Finite, normal-range values only (what the projection produces)."""
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)
    return np.ldexp(np.rint(m * 256.0) / 256.0, e)


def out_proj(o, wa, wb):
    """Grouped low-rank output projection (Hugging Face Transformers docs "DeepSeek-V4", section
    "Hybrid attention", grouped output projection; llm-atlas "DeepSeek-V4-Flash" config: o_groups,
    o_lora_rank, hidden_size). The heads are split into G consecutive groups; group g's concatenated
    head outputs (K = (H/G) D channels) go through wa[g] ([R, K]) to R channels; the G*R channels,
    stored in bf16, go through wb ([hidden, G*R]). fp64 from the bf16 inputs.
    Returns (z before its bf16 rounding [S, G*R], out [S, hidden]), both float64."""
    o_ = _as_f64(o)
    o_ = o_.reshape(o_.shape[0], -1)
    wa_, wb_ = _as_f64(wa), _as_f64(wb)
    G, R, K = wa_.shape
    assert o_.shape[1] == G * K and wb_.shape[1] == G * R
    z = np.concatenate([o_[:, g * K:(g + 1) * K] @ wa_[g].T for g in range(G)], axis=1)
    out = round_bf16(z) @ wb_.T
    return z, out


# ---- MXFP4 lightning-indexer operands (axbrief digest "Compressed attention and a new optimizer":
# MXFP4 on the indexer's query-key path; insight.ai.kr digest of the HF blog: the indexer is
# stored in FP4). The pages name the format without its details; it is taken as the OCP
# Microscaling one: blocks of 32 consecutive channels share an E8M0 scale 2^(e-127); elements are
# E2M1, rounded to nearest with ties to the even code and saturating at 6.

MXFP4_BLOCK = 32
E2M1_VALUES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])   # magnitude code 0..7


def _e2m1_round(q: np.ndarray) -> np.ndarray:
    """Magnitude codes (0..7) of |q| rounded to the nearest E2M1 value, ties to the even code,
    saturating at 6."""
    a = np.abs(q)
    code = np.zeros(a.shape, np.int64)
    for c in range(1, 8):   # walk up the grid: past the midpoint, or on it with an even upper code
        lo, hi = E2M1_VALUES[c - 1], E2M1_VALUES[c]
        mid = 0.5 * (lo + hi)
        up = (a > mid) | ((a == mid) & (c % 2 == 0))
        code = np.where(up & (code == c - 1), c, code)
    return code


def mxfp4_quantize(x):
    """x [..., d] (d a multiple of 32; bf16 or float values) -> (codes uint8 [..., d/2],
    scales uint8 [..., d/32]). Per block: amax = max |x|; e = 0 for amax = 0, else
    e = clamp(floor(log2 amax) - 2 + 127, 0, 254); element = E2M1 rounding of x / 2^(e-127), sign
    in bit 3 (never on a zero); channel 2i in the low nibble of byte i."""
    v = _as_f64(x)
    d = v.shape[-1]
    assert d % MXFP4_BLOCK == 0
    blocks = v.reshape(v.shape[:-1] + (d // MXFP4_BLOCK, MXFP4_BLOCK))
    amax = np.abs(blocks).max(axis=-1)
    with np.errstate(divide="ignore"):
        ex = np.floor(np.log2(np.where(amax > 0, amax, 1.0))).astype(np.int64)
    e = np.where(amax > 0, np.clip(ex - 2 + 127, 0, 254), 0)
    q = blocks / np.ldexp(1.0, e - 127)[..., None]
    mag = _e2m1_round(q)
    sign = (q < 0) & (mag > 0)
    nib = (mag | (sign.astype(np.int64) << 3)).reshape(v.shape)
    codes = (nib[..., 0::2] | (nib[..., 1::2] << 4)).astype(np.uint8)
    return codes, e.astype(np.uint8)


def mxfp4_dequantize(codes, scales) -> np.ndarray:
    """Inverse of the packing: values [..., 2 * codes.shape[-1]] float64 (exact)."""
    c = _np(codes, np.uint8).astype(np.int64)
    s = _np(scales, np.uint8).astype(np.int64)
    nib = np.stack([c & 15, c >> 4], axis=-1).reshape(c.shape[:-1] + (2 * c.shape[-1],))
    val = E2M1_VALUES[nib & 7] * np.where(nib & 8, -1.0, 1.0)
    d = val.shape[-1]
    blocks = val.reshape(val.shape[:-1] + (d // MXFP4_BLOCK, MXFP4_BLOCK))
    return (blocks * np.ldexp(1.0, s - 127)[..., None]).reshape(val.shape)


def _bf16_bits_exact(x: np.ndarray) -> np.ndarray:
    """bf16 bit patterns of float64 values that bf16 represents exactly (checked)."""
    f = np.ascontiguousarray(x.astype(np.float32))
    assert np.array_equal(f.astype(np.float64), x), "value not representable in fp32"
    bits = f.view(np.uint32)
    assert not np.any(bits & 0xFFFF), "value not representable in bf16"
    return (bits >> 16).astype(np.uint16)


def decode_index_topk_fp4(qc, qs, w, kc, ks, k: int, rows=None):
    """Decode indexer + top-k on MXFP4 operands: the indexer formula on the dequantised q^I
    [B, HI, dI] and k^I [B, T, dI] (every E2M1 value times a power of two is exact in bf16, so the
    bf16 oracle receives exactly these values)."""
    qv = _bf16_bits_exact(mxfp4_dequantize(qc, qs))
    kv = _bf16_bits_exact(mxfp4_dequantize(kc, ks))
    return decode_index_topk(qv, w, kv, k, rows=rows)


def index_topk_fp4(qc, qs, w, kc, ks, m: int, k: int, rows=None):
    """Prefill indexer + top-k on MXFP4 operands: the indexer formula on the dequantised q^I [S, HI, dI]
    and k^I [T, dI] (exact in bf16, see decode_index_topk_fp4)."""
    qv = _bf16_bits_exact(mxfp4_dequantize(qc, qs))
    kv = _bf16_bits_exact(mxfp4_dequantize(kc, ks))
    return index_topk(qv, kv, w, m, k, rows=rows)
