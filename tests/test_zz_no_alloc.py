"""csa_decode_noalloc: decode for callers that cannot allocate device memory.

Such callers (a runtime with no CUDA allocator of its own, or a serving loop that must not call
cudaMalloc while other work is in flight) get the decode step with its scratch taken from a fixed
array inside the library. Here it is called through the C ABI and compared with csa_decode, which
uses a caller-provided workspace, on two calls in a row (the second call finds the first call's
leftovers in the shared array). The file sorts last so a stop-at-first-failure run has already run
every other test."""
import ctypes

import pytest
import torch

import long_context_sparse_fwd_b200 as csa
from helpers import O_MAX_ABS, O_MEAN_ABS, check_close
from workloads import WORKLOADS, decode_inputs

pytestmark = pytest.mark.gpu

P_, I32, I64, F64, F32 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_double, ctypes.c_float


def noalloc_fn():
    f = csa.lib().csa_decode_noalloc
    f.restype = I32
    f.argtypes = [P_] * 10 + [I32, I32, I32, I64, I32, I32, I32, I32, I32, I64, F64, F64, F32, P_, P_, P_]
    return f


def ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def call_noalloc(y, wl, B, P, o, idx, cache):
    f = noalloc_fn()
    ent = (y["C"], None, None, None) if cache == "bf16" else (None, y["c8"], y["scale"], y["rope"])
    return f(ptr(y["q"]), ptr(y["qI"]), ptr(y["w"]), ptr(y["kI"]), *[ptr(e) for e in ent], ptr(y["win"]),
             ptr(y["sinks"]), B, wl.H, wl.D, wl.T, wl.HI, wl.dI, wl.topk, wl.W, wl.r, P, wl.theta_tok,
             wl.theta_cmp, 0.0, ptr(idx), ptr(o), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("wid,ctx,B,B2", [(3, 65536, 8, 6), (4, 131072, 4, 3), (3, 262144, 2, 1)])
def test_noalloc_decode_matches_decode(wid, ctx, B, B2):
    """Two calls in a row on different inputs (another seed and batch): each must equal csa_decode on
    the same inputs, so nothing the first call left in the shared array leaks into the second. The
    last case has 65536 entries per sequence, past the single-CTA top-k, so the chunked top-k's
    histograms, bitmap and candidates live in the shared array too."""
    for call, (seed_add, batch) in enumerate([(0, B), (17, B2)]):
        wl = WORKLOADS[wid].with_(ctx=ctx, seed=WORKLOADS[wid].seed + seed_add)
        y = decode_inputs(wl, device="cuda", batch=batch)
        P = wl.ctx - 1
        kw = dict(C=y["C"]) if wl.cache == "bf16" else dict(c8=y["c8"], c8_scale=y["scale"], c_rope=y["rope"])
        ref_o, ref_idx = csa.decode(y["q"], y["qI"], y["w"], y["kI"], y["win"], y["sinks"], P, wl.topk, wl.r,
                                    wl.theta_tok, wl.theta_cmp, **kw)
        torch.cuda.synchronize()
        o = torch.full_like(ref_o, float("nan"))
        idx = torch.full_like(ref_idx, -7)
        assert call_noalloc(y, wl, batch, P, o, idx, wl.cache) == 0, call
        torch.cuda.synchronize()
        check_close(o, ref_o.cpu().double().numpy(), O_MAX_ABS, O_MEAN_ABS, what=f"o (call {call})")
        assert torch.equal(idx, ref_idx), call


def test_noalloc_rejects_problems_beyond_its_scratch():
    limit = csa.lib().csa_decode_noalloc_max_scratch
    limit.restype = ctypes.c_size_t
    assert limit() == 16 << 20
    wl = WORKLOADS[3].with_(ctx=4096)
    y = decode_inputs(wl, device="cuda", batch=2)
    o = torch.empty(2, wl.H, wl.D, device="cuda")
    idx = torch.empty(2, wl.topk, dtype=torch.int32, device="cuda")
    # claims 64 sequences of 2^20 entries: 256 MiB of scores; refused before anything is launched
    f = noalloc_fn()
    rc = f(ptr(y["q"]), ptr(y["qI"]), ptr(y["w"]), ptr(y["kI"]), ptr(y["C"]), None, None, None, ptr(y["win"]),
           ptr(y["sinks"]), 64, wl.H, wl.D, 1 << 20, wl.HI, wl.dI, wl.topk, wl.W, wl.r, wl.ctx - 1, wl.theta_tok,
           wl.theta_cmp, 0.0, ptr(idx), ptr(o), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 5   # CSA_ERR_WORKSPACE
    # sizes whose byte counts would overflow are refused as invalid, also before anything is launched
    rc = f(ptr(y["q"]), ptr(y["qI"]), ptr(y["w"]), ptr(y["kI"]), ptr(y["C"]), None, None, None, ptr(y["win"]),
           ptr(y["sinks"]), 1 << 30, wl.H, wl.D, 1 << 40, wl.HI, wl.dI, wl.topk, wl.W, wl.r, wl.ctx - 1, wl.theta_tok,
           wl.theta_cmp, 0.0, ptr(idx), ptr(o), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 1   # CSA_ERR_INVALID_ARG
