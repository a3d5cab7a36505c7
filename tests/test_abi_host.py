"""CPU-only checks of the C ABI: the library loads, exports every call include/csa.h declares,
and rejects bad arguments on the host with the documented status before launching anything.

Every call below fails a host-side check, so no kernel is launched and no pointer is touched
(the fake pointers are never dereferenced)."""
import ctypes
import os
import re

import pytest

import long_context_sparse_fwd_b200 as csa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
INVALID, UNSUP, WS = 1, 2, 5


def declared_functions():
    names = []
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            names += re.findall(r"CSA_API\s+[\w\s\*]+?\b(\w+)\s*\(", src)
    return names


def test_library_exports_every_declared_call():
    names = declared_functions()
    assert len(names) >= 11
    L = ctypes.CDLL(csa.library_path())
    for n in names:
        assert hasattr(L, n), n
    assert csa.lib().csa_version().decode().startswith("csa-b200")


def test_status_strings():
    L = csa.lib()
    for code, name in [(0, "CSA_OK"), (1, "CSA_ERR_INVALID_ARG"), (2, "CSA_ERR_UNSUPPORTED"), (3, "CSA_ERR_CUDA"),
                       (4, "CSA_ERR_TIMEOUT"), (5, "CSA_ERR_WORKSPACE")]:
        assert L.csa_status_str(code).decode() == name


def test_workspace_sizes():
    assert csa.workspace_size("attend") == 256
    assert csa.workspace_size("hca_forward") == 256
    assert csa.workspace_size("index_topk", S=8192, T=2048) == 256 + 8192 * 2048 * 4   # no index shape given
    assert csa.workspace_size("index_topk", S=8192, T=8192, HI=64, dI=128, k=512) == 256 + 8192 * 8192 * 4
    assert csa.workspace_size("decode", B=64, T=32768, k=1024) >= 256 + 64 * 32768 * 4 + 64 * 1024 * 4


# The fake pointers below are only safe because every call fails a host check first; they are
# never handed to a machine with a GPU, where a check that regressed would launch a kernel on them.
no_gpu = pytest.mark.skipif(__import__("torch").cuda.is_available(), reason="fake-pointer checks run on CPU hosts only")

FAKE = ctypes.c_void_p(0x10000)      # 16-byte aligned, never dereferenced
MIS = ctypes.c_void_p(0x10002)       # misaligned


def compress(**kw):
    a = dict(kv=FAKE, gate=FAKE, b=FAKE, S=64, pos0=0, D=64, m=4, L=8, r=16, tc=160000.0, tt=10000.0, C=FAKE,
             kvr=FAKE)
    a.update(kw)
    return csa.lib().csa_compress(a["kv"], a["gate"], a["b"], a["S"], a["pos0"], a["D"], a["m"], a["L"], a["r"],
                                  a["tc"], a["tt"], a["C"], a["kvr"], None)


@no_gpu
def test_compress_rejects_bad_arguments():
    assert compress(S=-1) == INVALID
    assert compress(m=0) == INVALID
    assert compress(L=2) == INVALID            # window shorter than the stride
    assert compress(r=3) == INVALID            # odd rope dims
    assert compress(r=128) == INVALID          # rope dims beyond D
    assert compress(kv=None) == INVALID
    assert compress(C=None) == INVALID
    assert compress(tc=0.5) == INVALID
    assert compress(kv=MIS) == INVALID
    assert compress(D=60) == UNSUP
    assert compress(r=12) == UNSUP
    assert compress(L=8192, m=4096) == UNSUP
    assert compress(pos0=-1) == INVALID
    assert compress(pos0=1 << 41) == INVALID
    assert compress(S=3, pos0=5, C=None) == INVALID   # positions 5..7: entry 1 closes at 7 and there is no cache
    assert compress(S=2, pos0=4, C=None, kv=MIS) == INVALID


def attend(**kw):
    a = dict(q=FAKE, C=FAKE, kvr=FAKE, idx=FAKE, sinks=FAKE, S=64, pos0=0, H=8, D=128, T=16, k=4, W=8, r=32, m=4,
             tt=1e4, tc=1.6e5, sc=0.0, o=FAKE, ws=FAKE, wsb=256)
    a.update(kw)
    return csa.lib().csa_attend(a["q"], a["C"], a["kvr"], a["idx"], a["sinks"], a["S"], a["pos0"], a["H"], a["D"],
                                a["T"], a["k"], a["W"], a["r"], a["m"], a["tt"], a["tc"], a["sc"], a["o"], a["ws"],
                                a["wsb"], None)


@no_gpu
def test_attend_rejects_bad_arguments():
    assert attend(T=17) == INVALID             # more entries than floor(S/m)
    assert attend(T=17, pos0=4, D=96) == UNSUP  # 17 entries exist after a chunk at pos0 = 4: only D is wrong
    assert attend(T=18, pos0=4) == INVALID      # but not 18
    assert attend(pos0=-3) == INVALID
    assert attend(H=0) == INVALID
    assert attend(W=-1) == INVALID
    assert attend(k=0) == INVALID
    assert attend(idx=None) == INVALID
    assert attend(q=MIS) == INVALID
    assert attend(D=96) == UNSUP
    assert attend(k=5000) == UNSUP
    assert attend(ws=None) == WS
    assert attend(wsb=16) == WS
    assert attend(ws=ctypes.c_void_p(0x10010)) == INVALID   # workspace must be 256-byte aligned


@no_gpu
def test_index_topk_rejects_bad_arguments():
    L = csa.lib()
    f = lambda S=64, T=16, HI=4, dI=64, m=4, k=8, ws=FAKE, wsb=1 << 20, q=FAKE, pos0=0: L.csa_index_topk(
        q, FAKE, FAKE, S, pos0, T, HI, dI, m, k, FAKE, ws, wsb, None)
    assert f(T=17) == INVALID
    assert f(T=20, pos0=16, dI=48) == UNSUP     # 20 entries exist after a chunk at pos0 = 16: only dI is wrong
    assert f(T=21, pos0=16) == INVALID
    assert f(pos0=-1) == INVALID
    assert f(k=0) == INVALID
    assert f(q=None) == INVALID
    assert f(dI=48) == UNSUP
    assert f(wsb=100) == WS


@no_gpu
def test_decode_rejects_bad_arguments():
    L = csa.lib()

    def f(C=FAKE, c8=None, B=2, D=512, k=64, P=100, dI=128, wsb=1 << 24, T=256):
        return L.csa_decode(FAKE, FAKE, FAKE, FAKE, C, c8, None, None, FAKE, FAKE, B, 8, D, T, 4, dI, k, 8, 64,
                            P, 1e4, 1.6e5, 0.0, None, FAKE, FAKE, wsb, None)
    assert f(C=None) == INVALID                 # neither bf16 entries nor an FP8 cache
    assert f(P=-1) == INVALID
    assert f(D=96) == UNSUP
    assert f(dI=40) == UNSUP
    assert f(wsb=64) == WS
    assert f(T=1 << 41) == INVALID               # sizes that would overflow the workspace arithmetic
    assert f(B=1 << 30, T=1 << 30) == INVALID


def test_binding_refuses_cpu_tensors():
    import torch
    with pytest.raises(ValueError):
        csa.compress(torch.zeros(8, 8, dtype=torch.bfloat16), torch.zeros(8, 8, dtype=torch.bfloat16),
                     torch.zeros(8), 4, 8, 0, 1e4, 1e4)


@no_gpu
def test_later_calls_reject_bad_arguments():
    """hca_decode, swa_attend, csa_compress_append and csa_out_proj check their arguments on the host."""
    L = csa.lib()

    def hd(C=FAKE, B=2, D=512, T=100, P=1000, wsb=1 << 20):
        return L.hca_decode(FAKE, C, None, None, None, FAKE, FAKE, B, 64, D, T, 128, 64, P, 1e4, 1.6e5, 0.0, FAKE,
                            FAKE, wsb, None)
    assert hd(T=-1) == INVALID
    assert hd(P=-5) == INVALID
    assert hd(C=None) == INVALID                # entries but neither a bf16 nor an FP8 cache
    assert hd(D=96) == UNSUP
    assert hd(wsb=16) == WS

    assert L.swa_attend(FAKE, FAKE, FAKE, 64, 0, 8, 96, 128, 32, 1e4, 0.0, FAKE, FAKE, 256, None) == UNSUP
    assert L.swa_attend(FAKE, None, FAKE, 64, 0, 8, 128, 128, 32, 1e4, 0.0, FAKE, FAKE, 256, None) == INVALID
    assert L.swa_attend(FAKE, FAKE, FAKE, 64, -1, 8, 128, 128, 32, 1e4, 0.0, FAKE, FAKE, 256, None) == INVALID

    def ca(C=FAKE, D=512, Lw=8, P=7, Tcap=2):
        return L.csa_compress_append(FAKE, FAKE, FAKE, FAKE, FAKE, 2, D, 4, Lw, 64, P, 1.6e5, 1e4, C, None, None,
                                     None, Tcap, FAKE, 128, None)
    assert ca(Lw=2) == INVALID                  # pooling window shorter than the stride
    assert ca(P=11, Tcap=2) == INVALID          # entry 2 closes at P=11 but the cache holds two entries
    assert ca(C=None) == INVALID                # an entry closes and there is no cache to take it
    assert ca(D=520) == UNSUP

    def op(G=8, R=1024, hid=4096, wsb=256):
        return L.csa_out_proj(FAKE, FAKE, FAKE, 128, 64, 512, G, R, hid, FAKE, FAKE, FAKE, wsb, None)
    assert op(G=7) == INVALID                   # 64 heads do not split into 7 groups
    assert op(R=1000) == UNSUP                  # o_lora_rank not a multiple of 256
    assert op(hid=100) == UNSUP
    assert op(wsb=16) == WS


def test_fp4_calls_reject_bad_arguments():
    """csa_quantize_mxfp4 and csa_decode_fp4 check their arguments on the host, before any launch."""
    L = csa.lib()
    assert L.csa_quantize_mxfp4(FAKE, 4, 48, FAKE, FAKE, None) == INVALID     # 48 channels: not whole blocks
    assert L.csa_quantize_mxfp4(FAKE, -1, 64, FAKE, FAKE, None) == INVALID
    assert L.csa_quantize_mxfp4(None, 4, 64, FAKE, FAKE, None) == INVALID     # rows but no input
    assert L.csa_quantize_mxfp4(FAKE, 0, 64, None, None, None) == 0           # nothing to do

    def df(qc=FAKE, kc=FAKE, C=FAKE, B=2, T=100, HI=64, dI=128, k=64, wsb=1 << 24):
        return L.csa_decode_fp4(FAKE, qc, FAKE, FAKE, kc, FAKE, C, None, None, None, FAKE, FAKE, B, 64, 512, T, HI, dI,
                                k, 128, 64, 1000, 1e4, 1.6e5, 0.0, None, FAKE, FAKE, wsb, None)
    assert df(T=-1) == INVALID
    assert df(qc=None) == INVALID               # index query codes missing
    assert df(kc=None) == INVALID               # entries but no index key codes
    assert df(C=None) == INVALID                # entries but neither a bf16 nor an FP8 cache
    assert df(dI=96) == UNSUP                   # MXFP4 scan: d_I of 64 or 128

    def pf(qc=FAKE, kc=FAKE, S=64, pos0=0, T=16, HI=64, dI=128, k=8, qs=FAKE):
        return L.csa_index_topk_fp4(qc, qs, FAKE, kc, FAKE, S, pos0, T, HI, dI, 4, k, FAKE, FAKE, 256, None)
    assert pf(T=17) == INVALID                  # more entries than floor((pos0 + S) / m)
    assert pf(qc=None) == INVALID
    assert pf(qs=ctypes.c_void_p(0x10002)) == INVALID   # scales must be 4-byte aligned
    assert pf(dI=64) == UNSUP                   # the block-scaled prefill path takes d_I = 128
    assert pf(HI=128) == UNSUP
    assert df(HI=48) == UNSUP
    assert df(wsb=16) == WS
