"""GPU parity: every call of the C ABI against the fp64 oracle on the same seeded inputs.

Small cases cover several tiles and ragged tails in full; the V4-Flash-sized workloads are run in
the launch configuration the benchmark times and checked on sampled rows the oracle computes one
by one. Tolerances follow the acceptance rules (helpers.py)."""
import numpy as np
import pytest
import torch

import long_context_sparse_fwd_b200 as csa
import oracle
from helpers import C_MAX_ABS, O_MAX_ABS, O_MEAN_ABS, check_close, check_topk_sets, to_np
from workloads import WORKLOADS, attend_inputs, decode_inputs, prefill_inputs

pytestmark = pytest.mark.gpu
DEV = "cuda"


def dev(d):
    return {k: v.to(DEV) for k, v in d.items()}


def host(d):
    return {k: v.cpu() for k, v in d.items()}


def gen(fn, wl, **kw):
    """Draw inputs on the GPU (fast at full size); the oracle reads host copies of the same bits."""
    g = fn(wl, device=DEV, **kw)
    return g, host(g)


def sample_rows(S, n, seed, must=()):
    rng = np.random.default_rng(seed)
    rows = set(int(x) for x in rng.choice(S, size=min(n, S), replace=False))
    rows |= {r for r in must if 0 <= r < S}
    return np.array(sorted(rows), np.int64)


def bf16_rel_close(got, ref, what):
    got, ref = to_np(got), np.asarray(ref)
    err = np.abs(got - ref)
    bound = 2.0 ** -8 * np.abs(ref) + 1e-5
    assert (err <= bound).all(), f"{what}: {int((err > bound).sum())} values beyond bf16 rounding"


# ---- 1. compressor ---------------------------------------------------------------------------------

@pytest.mark.parametrize("wid,S", [(0, 1024), (0, 1030), (0, 3), (1, 8192), (2, 65536), (2, 65536 + 77)])
def test_compress(wid, S):
    wl = WORKLOADS[wid].with_(S=S)
    g, x = gen(prefill_inputs, wl, need_index=False, need_q=False)
    C, kvr = csa.compress(g["kv"], g["gate"], g["pos_bias"], wl.m, wl.L, wl.r, wl.theta_cmp, wl.theta_tok)
    torch.cuda.synchronize()
    Cr, kvrr = oracle.compress(x["kv"], x["gate"], x["pos_bias"], wl.m, wl.L, wl.r, wl.theta_cmp, wl.theta_tok)
    assert C.shape == (S // wl.m, wl.D)
    if S // wl.m:
        check_close(C, Cr, C_MAX_ABS, what="C")
        bf16_rel_close(C, Cr, "C")
    bf16_rel_close(kvr, kvrr, "kv_rot")


# ---- 2. indexer + top-k --------------------------------------------------------------------------------

@pytest.mark.parametrize("wid,S,nrows", [(0, 1024, None), (0, 1030, None), (0, 17, None), (1, 8192, 160)])
def test_index_topk(wid, S, nrows):
    wl = WORKLOADS[wid].with_(S=S)
    g, x = gen(prefill_inputs, wl, need_q=False)
    idx = csa.index_topk(g["qI"], g["kI"], g["w"], wl.m, wl.topk)
    torch.cuda.synchronize()
    rows = np.arange(S) if nrows is None else sample_rows(S, nrows, 7, must=range(S - 8, S))
    ridx, sc = oracle.index_topk(x["qI"], x["kI"], x["w"], wl.m, wl.topk, rows=rows)
    vis = [oracle.visible(t, wl.m, wl.T) for t in rows]
    exc = check_topk_sets(idx.cpu().numpy()[rows], ridx, sc, vis, wl.topk)
    assert len(exc) <= max(2, len(rows) // 50), f"too many near-tie exceptions: {exc[:5]}"
    # ascending order of the kept indices (the library's documented order)
    got = idx.cpu().numpy()
    for t in rows[:64]:
        kept = got[t][got[t] >= 0]
        assert (np.diff(kept) > 0).all()


@pytest.mark.parametrize("HI,dI,S,k", [(64, 128, 1030, 16), (32, 64, 777, 40), (128, 128, 600, 8),
                                        (16, 64, 5000, 300), (64, 128, 16384, 512), (64, 128, 20000, 512),
                                        (16, 64, 30000, 300), (64, 128, 40000, 1024), (64, 128, 65536, 512)])
def test_index_topk_shapes(HI, dI, S, k):
    """Tensor-core path shapes (N = 256 query-head columns), ragged query blocks and entry tiles, k above
    and below vis(t). Up to 4096 entries the scores of a group stay on chip whole; past that (S = 20000
    and up, to 16384 entries at S = 65536) they are ranked chunk by chunk against a running top-k."""
    wl = WORKLOADS[1].with_(S=S, HI=HI, dI=dI, topk=k)
    g, x = gen(prefill_inputs, wl, need_q=False)
    idx = csa.index_topk(g["qI"], g["kI"], g["w"], wl.m, wl.topk)
    torch.cuda.synchronize()
    rows = sample_rows(S, 96, 13, must=list(range(0, 9)) + [255, 256, 511, S - 2, S - 1])
    ridx, sc = oracle.index_topk(x["qI"], x["kI"], x["w"], wl.m, wl.topk, rows=rows)
    vis = [oracle.visible(t, wl.m, wl.T) for t in rows]
    exc = check_topk_sets(idx.cpu().numpy()[rows], ridx, sc, vis, wl.topk)
    assert len(exc) <= max(2, len(rows) // 50), f"too many near-tie exceptions: {exc[:5]}"


def test_index_topk_all_zero_ties():
    """Weights 0 make every score exactly 0: the k smallest visible indices win."""
    wl = WORKLOADS[0].with_(S=200)
    x = prefill_inputs(wl)
    x["w"] = torch.zeros_like(x["w"])
    g = dev(x)
    idx = csa.index_topk(g["qI"], g["kI"], g["w"], wl.m, wl.topk).cpu().numpy()
    for t in range(wl.S):
        n = min(wl.topk, (t + 1) // wl.m)
        assert idx[t][:n].tolist() == list(range(n)) and (idx[t][n:] == -1).all()



def test_index_topk_tc_all_zero_ties():
    """Tensor-core indexer with weights 0: every score is exactly 0, so each query keeps its k smallest
    visible indices; vis(t) from below k to far above the ranked-bin capacity (the crowded-bin path)."""
    wl = WORKLOADS[1].with_(S=3000, HI=64, dI=128, topk=64)
    g, x = gen(prefill_inputs, wl, need_q=False)
    g["w"] = torch.zeros_like(g["w"])
    idx = csa.index_topk(g["qI"], g["kI"], g["w"], wl.m, wl.topk).cpu().numpy()
    for t in [0, 3, 100, 255, 256, 260, 1000, 2047, 2048, 2100, 2999]:
        n = min(wl.topk, (t + 1) // wl.m)
        assert idx[t][:n].tolist() == list(range(n)) and (idx[t][n:] == -1).all(), t


def test_index_topk_tc_chunked_all_zero_ties():
    """Past 4096 entries (chunked ranking) with weights 0: every score is exactly 0 and each query keeps
    its k smallest visible indices, so ties across chunk boundaries go to the smaller index."""
    wl = WORKLOADS[1].with_(S=24000, HI=64, dI=128, topk=512)
    g, _ = gen(prefill_inputs, wl, need_q=False)
    g["w"] = torch.zeros_like(g["w"])
    idx = csa.index_topk(g["qI"], g["kI"], g["w"], wl.m, wl.topk).cpu().numpy()
    for t in [0, 2, 3, 2047, 2048, 11775, 11776, 12000, 16383, 23999]:
        n = min(wl.topk, (t + 1) // wl.m)
        assert idx[t][:n].tolist() == list(range(n)) and (idx[t][n:] == -1).all(), t


@pytest.mark.parametrize("classes,k,S", [(6, 128, 4100), (2, 300, 4100), (3, 256, 20004)])
def test_index_topk_tc_few_distinct_scores(classes, k, S):
    """Tensor-core indexer with k^I rows repeating `classes` vectors: each query's scores take only
    that many values, so its threshold value is shared by many entries (ranked directly, or the
    crowded-bin path past 512). The selection must equal the oracle's exactly."""
    wl = WORKLOADS[1].with_(S=S, HI=64, dI=128, topk=k)
    g, x = gen(prefill_inputs, wl, need_q=False)
    pattern = torch.arange(wl.T) % classes
    kI = x["kI"][:classes][pattern].contiguous()
    x["kI"] = kI
    g["kI"] = kI.to(DEV)
    idx = csa.index_topk(g["qI"], g["kI"], g["w"], wl.m, wl.topk).cpu().numpy()
    rows = sample_rows(wl.S, 48, 5, must=[0, 7, 1023, 2047, 2048, 4095, 4099, S - 1])
    ridx, _ = oracle.index_topk(x["qI"], x["kI"], x["w"], wl.m, wl.topk, rows=rows)
    for i, t in enumerate(rows):
        assert np.array_equal(idx[t], np.asarray(ridx[i], np.int32)), t

# ---- 3. CSA attention (oracle indices fed to the GPU) -----------------------------------------------------

@pytest.mark.parametrize("wid,S,nrows", [(0, 1024, None), (0, 1030, None), (0, 5, None), (1, 8192, 48)])
def test_csa_attend(wid, S, nrows):
    wl = WORKLOADS[wid].with_(S=S)
    gx, x = gen(prefill_inputs, wl)
    gy, y = gen(attend_inputs, wl)
    rows = np.arange(S) if nrows is None else sample_rows(S, nrows, 3, must=[0, 1, 2, 3, 127, 128, S - 1])
    ridx, _ = oracle.index_topk(x["qI"], x["kI"], x["w"], wl.m, wl.topk, rows=rows)
    idx_full = np.full((S, wl.topk), -1, np.int32)
    idx_full[rows] = ridx
    o = csa.attend(gx["q"], gy["C"], gy["kv_rot"], torch.tensor(idx_full, device=DEV), gx["sinks"], wl.m, wl.W,
                   wl.r, wl.theta_tok, wl.theta_cmp)
    torch.cuda.synchronize()
    ref = oracle.attend(x["q"], y["C"], y["kv_rot"], idx_full, x["sinks"], wl.m, wl.W, wl.r, wl.theta_tok,
                        wl.theta_cmp, rows=rows)
    check_close(o.cpu()[rows], ref, O_MAX_ABS, O_MEAN_ABS, what="o")


def test_csa_attend_reports_invisible_index():
    wl = WORKLOADS[0].with_(S=64)
    x = prefill_inputs(wl)
    y = attend_inputs(wl)
    idx = np.full((wl.S, wl.topk), -1, np.int32)
    idx[40, 0] = 3
    idx[40, 1] = 15          # not visible to t=40 (vis = 10): skipped and reported
    ws = torch.zeros(csa.workspace_size("attend"), dtype=torch.uint8, device=DEV)
    args = (x["q"].to(DEV), y["C"].to(DEV), y["kv_rot"].to(DEV))
    o = csa.attend(*args, torch.tensor(idx, device=DEV), x["sinks"].to(DEV), wl.m, wl.W, wl.r, wl.theta_tok,
                   wl.theta_cmp, workspace=ws)
    assert csa.get_device_status(ws) == 1
    idx[40, 1] = -1
    o2 = csa.attend(*args, torch.tensor(idx, device=DEV), x["sinks"].to(DEV), wl.m, wl.W, wl.r, wl.theta_tok,
                    wl.theta_cmp, workspace=ws)
    assert csa.get_device_status(ws) == 0
    assert torch.equal(o, o2)


# ---- 4. HCA attention -------------------------------------------------------------------------------------

@pytest.mark.parametrize("S,nrows", [(4096, 64), (1000, None)])
def test_hca_attend(S, nrows):
    wl = WORKLOADS[2].with_(S=S)
    gx, x = gen(prefill_inputs, wl)
    gy, y = gen(attend_inputs, wl)
    rows = np.arange(S) if nrows is None else sample_rows(S, nrows, 5, must=[0, 126, 127, 128, 255, S - 1])
    o = csa.hca_attend(gx["q"], gy["C"], gy["kv_rot"], gx["sinks"], wl.m, wl.W, wl.r, wl.theta_tok, wl.theta_cmp)
    torch.cuda.synchronize()
    ref = oracle.attend(x["q"], y["C"], y["kv_rot"], None, x["sinks"], wl.m, wl.W, wl.r, wl.theta_tok,
                        wl.theta_cmp, rows=rows)
    check_close(o.cpu()[rows], ref, O_MAX_ABS, O_MEAN_ABS, what="o")


# ---- 5. fused layer forward, end to end -----------------------------------------------------------------

@pytest.mark.parametrize("wid,S,nrows", [(0, 1024, None), (1, 8192, 24)])
def test_csa_forward_end_to_end(wid, S, nrows):
    wl = WORKLOADS[wid].with_(S=S)
    g, x = gen(prefill_inputs, wl)
    o, C, kvr, idx = csa.csa_forward(g["q"], g["kv"], g["gate"], g["pos_bias"], g["qI"], g["kI"], g["w"],
                                     g["sinks"], wl.m, wl.L, wl.topk, wl.W, wl.r, wl.theta_tok, wl.theta_cmp)
    torch.cuda.synchronize()
    rows = np.arange(S) if nrows is None else sample_rows(S, nrows, 9, must=[S - 1])
    Cr, kvrr = oracle.compress(x["kv"], x["gate"], x["pos_bias"], wl.m, wl.L, wl.r, wl.theta_cmp, wl.theta_tok)
    check_close(C, Cr, C_MAX_ABS, what="C")
    ridx, sc = oracle.index_topk(x["qI"], x["kI"], x["w"], wl.m, wl.topk, rows=rows)
    vis = [oracle.visible(t, wl.m, wl.T) for t in rows]
    exc = check_topk_sets(idx.cpu().numpy()[rows], ridx, sc, vis, wl.topk)
    keep = np.array([t for i, t in enumerate(rows) if i not in {e[0] for e in exc}])
    idx_full = np.full((S, wl.topk), -1, np.int32)
    idx_full[rows] = ridx
    ref = oracle.attend(x["q"], Cr, kvrr, idx_full, x["sinks"], wl.m, wl.W, wl.r, wl.theta_tok, wl.theta_cmp,
                        rows=keep)
    check_close(o.cpu()[keep], ref, O_MAX_ABS, O_MEAN_ABS, what="o")


def test_hca_forward_end_to_end():
    wl = WORKLOADS[2].with_(S=2048 + 100)
    g, x = gen(prefill_inputs, wl)
    o, C, kvr = csa.hca_forward(g["q"], g["kv"], g["gate"], g["pos_bias"], g["sinks"], wl.m, wl.L, wl.W, wl.r,
                                wl.theta_tok, wl.theta_cmp)
    torch.cuda.synchronize()
    rows = sample_rows(wl.S, 40, 4, must=[0, 127, 128, 1023, wl.S - 1])
    Cr, kvrr = oracle.compress(x["kv"], x["gate"], x["pos_bias"], wl.m, wl.L, wl.r, wl.theta_cmp, wl.theta_tok)
    check_close(C, Cr, C_MAX_ABS, what="C")
    ref = oracle.attend(x["q"], Cr, kvrr, None, x["sinks"], wl.m, wl.W, wl.r, wl.theta_tok, wl.theta_cmp, rows=rows)
    check_close(o.cpu()[rows], ref, O_MAX_ABS, O_MEAN_ABS, what="o")


@pytest.mark.parametrize("S", [65536, 16384 + 77])
def test_hca_forward_full_size(S):
    """The V4-Flash HCA prefill layer at its own size (65536 tokens: up to 512 pooled entries, eight
    64-key entry blocks per query) and at 16461 tokens (a ragged last entry block), in the launch
    configuration the benchmark times, on sampled rows: the last 64, both sides of window closes
    (128 j - 1 and 128 j) and random rows. Rows are independent once the entries exist."""
    wl = WORKLOADS[2].with_(S=S)
    g, x = gen(prefill_inputs, wl)
    o, C, kvr = csa.hca_forward(g["q"], g["kv"], g["gate"], g["pos_bias"], g["sinks"], wl.m, wl.L, wl.W, wl.r,
                                wl.theta_tok, wl.theta_cmp)
    torch.cuda.synchronize()
    must = list(range(S - 64, S)) + [128 * j - 1 for j in (1, 2, 3, 64, 128, 255, 256, 511)] + \
        [128 * j for j in (1, 2, 64, 128, 256, 500)]
    rows = sample_rows(S, 64, 21, must=must)
    Cr, kvrr = oracle.compress(x["kv"], x["gate"], x["pos_bias"], wl.m, wl.L, wl.r, wl.theta_cmp, wl.theta_tok)
    check_close(C, Cr, C_MAX_ABS, what="C")
    bf16_rel_close(kvr[torch.as_tensor(rows, device=DEV)], kvrr[rows], "kv_rot")
    ref = oracle.attend(x["q"], Cr, kvrr, None, x["sinks"], wl.m, wl.W, wl.r, wl.theta_tok, wl.theta_cmp, rows=rows)
    got = o[torch.as_tensor(rows, device=DEV)].cpu()
    check_close(got, ref, O_MAX_ABS, O_MEAN_ABS, what="o")


# ---- 5b. prefill in chunks (state carried across calls: pos0) -------------------------------------------

def _chunked_csa(wl, g, bounds):
    """csa_forward over the chunks [bounds[i], bounds[i+1]) of one sequence, the caches (C, kv_rot)
    carried from chunk to chunk; returns (o, C, kv_rot, idx) over all positions."""
    S, D, m = wl.S, wl.D, wl.m
    C = torch.full((S // m, D), float("nan"), dtype=torch.bfloat16, device=DEV)
    kvr = torch.full((S, D), float("nan"), dtype=torch.bfloat16, device=DEV)
    o = torch.empty(S, wl.H, D, dtype=torch.float32, device=DEV)
    idx = torch.empty(S, wl.topk, dtype=torch.int32, device=DEV)
    for a, b in zip(bounds[:-1], bounds[1:]):
        n = b
        csa.csa_forward(g["q"][a:b], g["kv"][:n], g["gate"][:n], g["pos_bias"], g["qI"][a:b], g["kI"][:n // m],
                        g["w"][a:b], g["sinks"], m, wl.L, wl.topk, wl.W, wl.r, wl.theta_tok, wl.theta_cmp,
                        out=(o[a:b], C[:n // m], kvr[:n], idx[a:b]), pos0=a)
    torch.cuda.synchronize()
    return o, C, kvr, idx


@pytest.mark.parametrize("wid,bounds,nrows", [(1, (0, 4096, 8192), 24), (0, (0, 333, 601, 1030), None)])
def test_csa_forward_chunked_equals_one_shot(wid, bounds, nrows):
    """A prefill split into chunks (V4-Flash shapes 4096 + 4096 on the tensor-core kernels; the tiny
    layer in chunks starting inside stride blocks on the general kernels) gives bit for bit the
    one-shot results: entries, window rows, top-k sets and outputs; the last chunk's rows also match
    the oracle's one-shot prefill."""
    wl = WORKLOADS[wid].with_(S=bounds[-1])
    g, x = gen(prefill_inputs, wl)
    o1, C1, kvr1, idx1 = csa.csa_forward(g["q"], g["kv"], g["gate"], g["pos_bias"], g["qI"], g["kI"], g["w"],
                                         g["sinks"], wl.m, wl.L, wl.topk, wl.W, wl.r, wl.theta_tok, wl.theta_cmp)
    o, C, kvr, idx = _chunked_csa(wl, g, bounds)
    assert torch.equal(C, C1) and torch.equal(kvr, kvr1)
    assert torch.equal(idx, idx1)
    assert torch.equal(o, o1)
    a = bounds[-2]
    rows = np.arange(a, wl.S) if nrows is None else sample_rows(wl.S - a, nrows, 19, must=[0, wl.S - a - 1]) + a
    ridx, sc = oracle.index_topk(x["qI"], x["kI"], x["w"], wl.m, wl.topk, rows=rows)
    vis = [oracle.visible(t, wl.m, wl.T) for t in rows]
    exc = check_topk_sets(idx.cpu().numpy()[rows], ridx, sc, vis, wl.topk)
    keep = np.array([t for i, t in enumerate(rows) if i not in {e[0] for e in exc}])
    Cr, kvrr = oracle.compress(x["kv"], x["gate"], x["pos_bias"], wl.m, wl.L, wl.r, wl.theta_cmp, wl.theta_tok)
    idx_full = np.full((wl.S, wl.topk), -1, np.int32)
    idx_full[rows] = ridx
    ref = oracle.attend(x["q"], Cr, kvrr, idx_full, x["sinks"], wl.m, wl.W, wl.r, wl.theta_tok, wl.theta_cmp,
                        rows=keep)
    check_close(o.cpu()[keep], ref, O_MAX_ABS, O_MEAN_ABS, what="o")


def test_hca_forward_chunked_equals_one_shot():
    """HCA prefill in two chunks, the second starting inside a 128-token window (entry 7 pools positions
    896..1023, 104 of them from the first chunk): bit for bit the one-shot results."""
    wl = WORKLOADS[2].with_(S=4096 + 77)
    g, _ = gen(prefill_inputs, wl)
    o1, C1, kvr1 = csa.hca_forward(g["q"], g["kv"], g["gate"], g["pos_bias"], g["sinks"], wl.m, wl.L, wl.W, wl.r,
                                   wl.theta_tok, wl.theta_cmp)
    S, D, m = wl.S, wl.D, wl.m
    C = torch.full((S // m, D), float("nan"), dtype=torch.bfloat16, device=DEV)
    kvr = torch.full((S, D), float("nan"), dtype=torch.bfloat16, device=DEV)
    o = torch.empty(S, wl.H, D, dtype=torch.float32, device=DEV)
    for a, b in ((0, 1000), (1000, S)):
        csa.hca_forward(g["q"][a:b], g["kv"][:b], g["gate"][:b], g["pos_bias"], g["sinks"], m, wl.L, wl.W, wl.r,
                        wl.theta_tok, wl.theta_cmp, out=(o[a:b], C[:b // m], kvr[:b]), pos0=a)
    torch.cuda.synchronize()
    assert torch.equal(C, C1) and torch.equal(kvr, kvr1) and torch.equal(o, o1)


def test_index_topk_workspace_is_status_word_on_the_tensor_core_path():
    """The fused tensor-core indexer keeps its scores on chip: its workspace is the status word only."""
    assert csa.workspace_size("index_topk", S=8192, T=2048, HI=64, dI=128, k=512) == 256
    assert csa.workspace_size("csa_forward", S=8192, T=2048, HI=64, dI=128, k=512) == 256
    # past 4096 entries as well: ranked chunk by chunk on chip, no S x T scores
    assert csa.workspace_size("index_topk", S=65536, T=16384, HI=64, dI=128, k=512) == 256


def test_forward_is_deterministic():
    wl = WORKLOADS[0]
    g = prefill_inputs(wl, device=DEV)
    run = lambda: csa.csa_forward(g["q"], g["kv"], g["gate"], g["pos_bias"], g["qI"], g["kI"], g["w"], g["sinks"],
                                  wl.m, wl.L, wl.topk, wl.W, wl.r, wl.theta_tok, wl.theta_cmp)
    a, b = run(), run()
    for u, v in zip(a, b):
        assert torch.equal(u, v)


# ---- 6. decode --------------------------------------------------------------------------------------------

def _decode_check(wl, batch, seqs):
    y = decode_inputs(wl, device=DEV, batch=batch)
    P = wl.ctx - 1
    kw = dict(C=y["C"]) if wl.cache == "bf16" else dict(c8=y["c8"], c8_scale=y["scale"], c_rope=y["rope"])
    o, idx = csa.decode(y["q"], y["qI"], y["w"], y["kI"], y["win"], y["sinks"], P, wl.topk, wl.r, wl.theta_tok,
                        wl.theta_cmp, **kw)
    torch.cuda.synchronize()
    seqs = np.asarray(seqs, np.int64)
    h = {k: v[seqs].cpu() if v.dim() > 1 else v.cpu() for k, v in y.items()}
    ridx, sc = oracle.decode_index_topk(h["qI"], h["w"], h["kI"], wl.topk)
    exc = check_topk_sets(idx.cpu().numpy()[seqs], ridx, sc, [wl.T] * len(seqs), wl.topk)
    keep = [i for i in range(len(seqs)) if i not in {e[0] for e in exc}]
    hk = {k: (v[keep] if v.dim() > 1 else v) for k, v in h.items()}
    kwr = dict(C=hk["C"]) if wl.cache == "bf16" else dict(c8=hk["c8"], c8_scale=hk["scale"], c_rope=hk["rope"])
    ref = oracle.decode_attend(hk["q"], hk["win"], ridx[keep], hk["sinks"], P, wl.r, wl.theta_tok, wl.theta_cmp, **kwr)
    check_close(o.cpu()[seqs[keep]], ref, O_MAX_ABS, O_MEAN_ABS, what="o")


def test_decode_bf16_small():
    _decode_check(WORKLOADS[3].with_(ctx=8192 + 4), batch=3, seqs=[0, 1, 2])


def test_decode_ctx128k_full_batch():
    _decode_check(WORKLOADS[3], batch=None, seqs=[0, 37, 63])


def test_decode_fp8_ctx1m():
    _decode_check(WORKLOADS[4], batch=None, seqs=[0, 7])


@pytest.mark.parametrize("batch", [37, 20])
def test_decode_split_counts(batch):
    """Batches that spread each sequence's key blocks over 4 and 7 CTAs (148 / B splits), so the split combine
    runs its 4- and 8-row instances; selections and outputs against the oracle on sampled sequences."""
    _decode_check(WORKLOADS[3].with_(ctx=4 * 4096 + 3), batch=batch, seqs=[0, batch // 2, batch - 1])


def test_decode_short_history():
    """P < W-1: window rows at negative positions are ignored; k > T pads with -1."""
    wl = WORKLOADS[3].with_(ctx=40, topk=16, W=128)
    _decode_check(wl, batch=2, seqs=[0, 1])


def _decode_index_only(y, wl):
    """Run csa_decode and return the selected indices (attention output unused)."""
    P = wl.ctx - 1
    kw = dict(C=y["C"]) if wl.cache == "bf16" else dict(c8=y["c8"], c8_scale=y["scale"], c_rope=y["rope"])
    _, idx = csa.decode(y["q"], y["qI"], y["w"], y["kI"], y["win"], y["sinks"], P, wl.topk, wl.r, wl.theta_tok,
                        wl.theta_cmp, **kw)
    torch.cuda.synchronize()
    return idx.cpu().numpy()


@pytest.mark.parametrize("ctx", [4 * 20000, 4 * 40000])
def test_decode_topk_all_scores_tied(ctx):
    """Index weights of zero make every score +0: the top-k is the k smallest indices (ties go to the
    smaller index), taken through the crowded-bin path since T far exceeds the candidate capacity.
    T = 20000 selects within one CTA per sequence, T = 40000 through the chunked kernels."""
    wl = WORKLOADS[3].with_(ctx=ctx, topk=1024)
    y = decode_inputs(wl, device=DEV, batch=2)
    y["w"] = torch.zeros_like(y["w"])
    idx = _decode_index_only(y, wl)
    want = np.arange(wl.topk, dtype=np.int32)
    for b in range(2):
        assert np.array_equal(idx[b], want)


@pytest.mark.parametrize("ctx,classes", [(4 * 8192, 5), (4 * 40000, 7)])
def test_decode_topk_few_distinct_scores(ctx, classes):
    """k^I rows repeat a few distinct vectors, so scores take `classes` values and the threshold value
    is shared by many entries (directly ranked, or the crowded-bin fallback past its capacity): the
    selection must equal the oracle's exactly, in ascending order."""
    wl = WORKLOADS[3].with_(ctx=ctx, topk=1024)
    y = decode_inputs(wl, device=DEV, batch=2)
    kI = y["kI"]
    base = kI[:, :classes].clone()
    pattern = torch.arange(wl.T, device=kI.device) % classes
    y["kI"] = base[:, pattern].contiguous()
    idx = _decode_index_only(y, wl)
    h = {k: v.cpu() for k, v in y.items()}
    ridx, _ = oracle.decode_index_topk(h["qI"], h["w"], h["kI"], wl.topk)
    for b in range(2):
        assert np.array_equal(idx[b], np.asarray(ridx[b], np.int32)), b
        assert np.all(np.diff(idx[b][idx[b] >= 0]) > 0)


# ---- FP4 (MXFP4) lightning indexer, decode --------------------------------------------------------------

def test_quantize_mxfp4_matches_oracle():
    """bf16 rows of mixed magnitudes (row scales 2^-40 .. 2^40), an all-zero block and exact E2M1
    midpoints: codes and scales bit-exact with the oracle."""
    g = torch.Generator().manual_seed(11)
    x = torch.randn(300, 128, generator=g, dtype=torch.float64)
    x *= torch.pow(2.0, torch.randint(-40, 41, (300, 1), generator=g).double())
    x[5, 32:64] = 0.0
    x[6, :8] = torch.tensor([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 7.0], dtype=torch.float64)
    x[6, 8:32] = 0.0
    xb = x.to(torch.bfloat16)
    codes, scales = csa.quantize_mxfp4(xb.to(DEV))
    torch.cuda.synchronize()
    rc, rs = oracle.mxfp4_quantize(xb)
    assert np.array_equal(scales.cpu().numpy(), rs)
    assert np.array_equal(codes.cpu().numpy(), rc)


def _decode_fp4_check(wl, batch, seqs):
    y = decode_inputs(wl, device=DEV, batch=batch)
    P = wl.ctx - 1
    qc, qs = csa.quantize_mxfp4(y["qI"])
    kc, ks = csa.quantize_mxfp4(y["kI"])
    kw = dict(C=y["C"]) if wl.cache == "bf16" else dict(c8=y["c8"], c8_scale=y["scale"], c_rope=y["rope"])
    o, idx = csa.decode_fp4(y["q"], qc, qs, y["w"], kc, ks, y["win"], y["sinks"], P, wl.topk, wl.r, wl.theta_tok,
                            wl.theta_cmp, **kw)
    torch.cuda.synchronize()
    seqs = np.asarray(seqs, np.int64)
    h = {k: v[seqs].cpu() if v.dim() > 1 else v.cpu() for k, v in y.items()}
    rq = oracle.mxfp4_quantize(h["qI"])
    rk = oracle.mxfp4_quantize(h["kI"])
    assert np.array_equal(qc.cpu().numpy()[seqs], rq[0]) and np.array_equal(kc.cpu().numpy()[seqs], rk[0])
    ridx, sc = oracle.decode_index_topk_fp4(rq[0], rq[1], h["w"], rk[0], rk[1], wl.topk)
    gidx = idx.cpu().numpy()[seqs]
    exc = check_topk_sets(gidx, ridx, sc, [wl.T] * len(seqs), wl.topk)
    assert len(exc) <= 1, f"near-tie exceptions in {len(exc)} sequences"
    assert all(np.all(np.diff(r[r >= 0]) > 0) for r in gidx)
    # the attention over the selection the GPU made (its sets are the oracle's up to near-ties)
    kwr = dict(C=h["C"]) if wl.cache == "bf16" else dict(c8=h["c8"], c8_scale=h["scale"], c_rope=h["rope"])
    ref = oracle.decode_attend(h["q"], h["win"], gidx, h["sinks"], P, wl.r, wl.theta_tok, wl.theta_cmp, **kwr)
    check_close(o.cpu()[seqs], ref, O_MAX_ABS, O_MEAN_ABS, what="o")


def test_decode_fp4_small():
    """MXFP4 indexer, ragged last tile (T = 2049), one CTA per sequence for the top-k."""
    _decode_fp4_check(WORKLOADS[3].with_(ctx=4 * 2049 + 3), batch=3, seqs=[0, 1, 2])


def test_decode_fp4_ctx128k():
    """MXFP4 indexer at the 128K decode size (64 sequences of 32768 entries), sampled sequences."""
    _decode_fp4_check(WORKLOADS[3], batch=None, seqs=[0, 41, 63])


def test_decode_fp4_chunked_topk_fp8_cache():
    """MXFP4 indexer past 32768 entries (chunked top-k) with the FP8 entry cache."""
    _decode_fp4_check(WORKLOADS[4].with_(ctx=4 * 40000 + 1, B=2), batch=None, seqs=[0, 1])


@pytest.mark.parametrize("HI,ctx,spread", [(64, 4 * 2052, 0), (16, 4 * 4100, 0), (32, 4 * 1000 + 2, 0),
                                             (64, 4 * 8192, 40)])
def test_decode_fp4_block_scaled_mma(HI, ctx, spread):
    """The MXFP4 scan on the block-scaled MMA (d_I = 128, HI <= 64, T a multiple of 4): a ragged last
    tile, N = 16 and 32 query-head columns, and k^I rows whose magnitudes span 2^-spread .. 2^spread so
    the E8M0 scales cover a wide range; selections equal the oracle's on the dequantised operands."""
    wl = WORKLOADS[3].with_(ctx=ctx, HI=HI, topk=256)
    assert wl.T % 4 == 0
    y = decode_inputs(wl, device=DEV, batch=3)
    if spread:
        g = torch.Generator(device=DEV).manual_seed(23)
        mag = torch.pow(2.0, torch.randint(-spread, spread + 1, (3, wl.T, 1), generator=g, device=DEV).float())
        y["kI"] = (y["kI"].float() * mag).to(torch.bfloat16)
    _decode_fp4_from(wl, y, seqs=[0, 1, 2])


def _decode_fp4_from(wl, y, seqs):
    P = wl.ctx - 1
    qc, qs = csa.quantize_mxfp4(y["qI"])
    kc, ks = csa.quantize_mxfp4(y["kI"])
    o, idx = csa.decode_fp4(y["q"], qc, qs, y["w"], kc, ks, y["win"], y["sinks"], P, wl.topk, wl.r, wl.theta_tok,
                            wl.theta_cmp, C=y["C"])
    torch.cuda.synchronize()
    seqs = np.asarray(seqs, np.int64)
    h = {k: v[seqs].cpu() if v.dim() > 1 else v.cpu() for k, v in y.items()}
    rq = oracle.mxfp4_quantize(h["qI"])
    rk = oracle.mxfp4_quantize(h["kI"])
    ridx, sc = oracle.decode_index_topk_fp4(rq[0], rq[1], h["w"], rk[0], rk[1], wl.topk)
    gidx = idx.cpu().numpy()[seqs]
    exc = check_topk_sets(gidx, ridx, sc, [wl.T] * len(seqs), wl.topk)
    assert len(exc) <= 1, f"near-tie exceptions in {len(exc)} sequences"
    ref = oracle.decode_attend(h["q"], h["win"], gidx, h["sinks"], P, wl.r, wl.theta_tok, wl.theta_cmp, C=h["C"])
    check_close(o.cpu()[seqs], ref, O_MAX_ABS, O_MEAN_ABS, what="o")


@pytest.mark.parametrize("HI,S,k,pos0,nrows", [(64, 8192, 512, 0, 160), (16, 1030, 64, 0, None),
                                                (32, 2048 + 37, 128, 0, 96), (64, 3000, 256, 1000, 96)])
def test_index_topk_fp4_prefill(HI, S, k, pos0, nrows):
    """Prefill lightning indexer on MXFP4 operands (block-scaled MMA, fused top-k): V4-Flash shapes at
    S = 8192 (sampled rows), N = 16 and 32 head columns with ragged entry tiles, and a chunk at pos0 > 0
    against the whole sequence's entries; sets equal the oracle's on the dequantised operands."""
    wl = WORKLOADS[1].with_(S=S, HI=HI, topk=k)
    g, x = gen(prefill_inputs, wl, need_q=False)
    qc, qs = csa.quantize_mxfp4(g["qI"].reshape(S * HI, wl.dI))
    kc, ks = csa.quantize_mxfp4(g["kI"])
    qc, qs = qc.reshape(S, HI, wl.dI // 2), qs.reshape(S, HI, wl.dI // 32)
    a = pos0
    idx = csa.index_topk_fp4(qc[a:], qs[a:], g["w"][a:], kc, ks, wl.m, k, pos0=a)
    torch.cuda.synchronize()
    rows = np.arange(a, S) if nrows is None else sample_rows(S - a, nrows, 29, must=[0, 1, S - a - 1]) + a
    hq, hk = (qc.cpu(), qs.cpu()), (kc.cpu(), ks.cpu())
    ridx, sc = oracle.index_topk_fp4(hq[0], hq[1], x["w"], hk[0], hk[1], wl.m, k, rows=rows)
    vis = [oracle.visible(t, wl.m, wl.T) for t in rows]
    exc = check_topk_sets(idx.cpu().numpy()[rows - a], ridx, sc, vis, k)
    assert len(exc) <= max(2, len(rows) // 50), f"too many near-tie exceptions: {exc[:5]}"


# ---- 7. HCA decode and the sliding-window-only layer ----------------------------------------------------

# HCA at 1M context: m' = 128 pools 1,048,576 tokens into T = 8192 entries, all attended densely
HCA_DEC = WORKLOADS[3].with_(name="hca_decode_b8_ctx1m", m=128, L=128, ctx=1 << 20, B=8, topk=0, seed=5)


def _hca_decode_check(wl, batch, seqs, entries=True):
    y = decode_inputs(wl, device=DEV, batch=batch)
    P = wl.ctx - 1
    if not entries:
        kw, T = {}, 0
    elif wl.cache == "bf16":
        kw, T = dict(C=y["C"]), wl.T
    else:
        kw, T = dict(c8=y["c8"], c8_scale=y["scale"], c_rope=y["rope"]), wl.T
    o = csa.hca_decode(y["q"], y["win"], y["sinks"], P, wl.r, wl.theta_tok, wl.theta_cmp, **kw)
    torch.cuda.synchronize()
    seqs = np.asarray(seqs, np.int64)
    h = {k: v[seqs].cpu() if v.dim() > 1 else v.cpu() for k, v in y.items()}
    idx = np.tile(np.arange(T, dtype=np.int32), (len(seqs), 1))
    if not entries:
        kwr = dict(C=h["C"][:, :0]) if "C" in h else dict(c8=h["c8"][:, :0], c8_scale=h["scale"][:, :0],
                                                          c_rope=h["rope"][:, :0])
    elif wl.cache == "bf16":
        kwr = dict(C=h["C"])
    else:
        kwr = dict(c8=h["c8"], c8_scale=h["scale"], c_rope=h["rope"])
    ref = oracle.decode_attend(h["q"], h["win"], idx, h["sinks"], P, wl.r, wl.theta_tok, wl.theta_cmp, **kwr)
    check_close(o.cpu()[seqs], ref, O_MAX_ABS, O_MEAN_ABS, what="o")


def test_hca_decode_bf16_ctx1m():
    _hca_decode_check(HCA_DEC, batch=None, seqs=[0, 5])


def test_hca_decode_fp8_ctx1m():
    _hca_decode_check(HCA_DEC.with_(cache="fp8"), batch=4, seqs=[1, 3])


def test_hca_decode_short_history():
    """Three pooled entries and a window reaching below position 0."""
    _hca_decode_check(HCA_DEC.with_(ctx=128 * 3 + 50), batch=3, seqs=[0, 1, 2])


def test_swa_decode():
    """The sliding-window-only layer's decode: hca_decode with no entry cache."""
    _hca_decode_check(HCA_DEC.with_(ctx=5000), batch=4, seqs=[0, 3], entries=False)


@pytest.mark.parametrize("wid,S,nrows", [(0, 1030, None), (1, 4096, 64)])
def test_swa_attend(wid, S, nrows):
    """Sliding-window-only prefill (no compressed entries): the general path (tiny heads) and the
    tensor-core path (64 heads x 512), against the oracle's attention with an empty entry set."""
    wl = WORKLOADS[wid].with_(S=S)
    g, x = gen(prefill_inputs, wl, need_index=False)
    a = attend_inputs(wl, device=DEV)
    o = csa.swa_attend(g["q"], a["kv_rot"], g["sinks"], wl.W, wl.r, wl.theta_tok)
    torch.cuda.synchronize()
    rows = None if nrows is None else sample_rows(S, nrows, 11, must=[0, 1, 127, 128, S - 1])
    ah = host(a)
    ref = oracle.attend(x["q"], ah["C"][:0], ah["kv_rot"], None, x["sinks"], 1, wl.W, wl.r, wl.theta_tok,
                        wl.theta_tok, rows=rows)
    got = o.cpu() if rows is None else o.cpu()[rows]
    check_close(got, ref, O_MAX_ABS, O_MEAN_ABS, what="o")


# ---- 8. the compressor's decode step ------------------------------------------------------------------

def _append_history(wl, B, S, fp8=False):
    """B independent histories of S tokens appended one position at a time; returns host inputs and
    the device caches."""
    xs = [prefill_inputs(wl.with_(S=S, seed=wl.seed + 100 * b), need_index=False, need_q=False) for b in range(B)]
    kv = torch.stack([x["kv"] for x in xs])
    gate = torch.stack([x["gate"] for x in xs])
    bias = xs[0]["pos_bias"]
    T, D, r, L, W = S // wl.m, wl.D, wl.r, wl.L, wl.W
    kv_d, gate_d, bias_d = kv.to(DEV), gate.to(DEV), bias.to(DEV)
    state_x = torch.empty(B, L, D, dtype=torch.bfloat16, device=DEV)
    state_g = torch.empty(B, L, D, dtype=torch.bfloat16, device=DEV)
    win = torch.zeros(B, W, D, dtype=torch.bfloat16, device=DEV)
    cache = {}
    if fp8:
        cache = dict(c8=torch.zeros(B, T, D - r, dtype=torch.uint8, device=DEV),
                     c8_scale=torch.zeros(B, T, dtype=torch.float32, device=DEV),
                     c_rope=torch.zeros(B, T, r, dtype=torch.bfloat16, device=DEV))
    else:
        cache = dict(C=torch.zeros(B, T, D, dtype=torch.bfloat16, device=DEV))
    for P in range(S):
        csa.compress_append(kv_d[:, P].contiguous(), gate_d[:, P].contiguous(), bias_d, state_x, state_g, P, wl.m,
                            r, wl.theta_cmp, wl.theta_tok, win=win, **cache)
    torch.cuda.synchronize()
    refs = [oracle.compress(kv[b], gate[b], bias, wl.m, wl.L, r, wl.theta_cmp, wl.theta_tok) for b in range(B)]
    return kv, gate, bias, win, cache, refs


@pytest.mark.parametrize("m,L,S,B", [(4, 8, 70, 3), (128, 128, 300, 2)])
def test_compress_append_matches_prefill_compressor(m, L, S, B):
    """Token-by-token decode steps leave in the cache exactly the prefill compressor's entries over the
    same history (CSA overlapping windows, HCA non-overlapping), and in the window ring the rows of the
    last W positions rotated at their own positions."""
    wl = WORKLOADS[1].with_(m=m, L=L)
    kv, gate, bias, win, cache, refs = _append_history(wl, B, S)
    T, W = S // m, wl.W
    for b in range(B):
        Cr, kvr = refs[b]
        check_close(cache["C"][b].float().cpu(), Cr[:T], C_MAX_ABS, what="C")
        bf16_rel_close(cache["C"][b].float().cpu(), Cr[:T], "C")
        for pos in range(max(0, S - W), S):
            bf16_rel_close(win[b, (W - 1 - pos) % W].float().cpu(), kvr[pos], "window row")


def _fp8_codes_match(codes, ref_nope, scale, what, max_ties):
    """GPU codes against the oracle's E4M3 encoding of ref / scale (the GPU's own scale, so both take
    the rounding decision on the same quotient). Where the quotient lies within 1e-5 relative of a
    rounding boundary between two codes the two sides' pooled values (fp32 against fp64) may fall on
    different sides: either neighbouring code is accepted there, and such ties are counted."""
    q = np.asarray(ref_nope, np.float64) / np.asarray(scale, np.float64)[:, None]
    lo = oracle.e4m3_encode((q * (1 - 1e-5)).astype(np.float32))
    hi = oracle.e4m3_encode((q * (1 + 1e-5)).astype(np.float32))
    want = oracle.e4m3_encode(q.astype(np.float32))
    tie = lo != hi
    ok = (codes == want) | (tie & ((codes == lo) | (codes == hi)))
    assert ok.all(), f"{what}: {int((~ok).sum())} codes differ from the oracle's encoding"
    assert int(tie.sum()) <= max_ties, f"{what}: {int(tie.sum())} near-boundary quotients"


def test_compress_append_fp8_codes_exact():
    """With m = L = 1 an entry is its token exactly (a one-position softmax has weight 1), so the FP8
    codes and scales must equal the oracle's bit for bit: scale = amax/448 in binary32, codes the
    nearest E4M3 value of x / scale with ties to the even code. Row 0 of each sequence is crafted so
    its scale is exactly 1 and its elements sit on E4M3 rounding midpoints."""
    wl = WORKLOADS[1].with_(m=1, L=1)
    B, S, D, r = 2, 6, wl.D, wl.r
    xs = [prefill_inputs(wl.with_(S=S, seed=wl.seed + 100 * b), need_index=False, need_q=False) for b in range(B)]
    kv = torch.stack([x["kv"] for x in xs]).float()
    mids = [448.0, 1.0625, 1.1875, -1.0625, -1.1875, 2.0 ** -10, 3 * 2.0 ** -10, 0.0, 13.0, 15.0, 240.0, -416.0]
    for b in range(B):
        kv[b, 0, :D - r] = torch.tensor(mids * ((D - r) // len(mids)) + mids[:(D - r) % len(mids)])
    kv = kv.to(torch.bfloat16)
    gate = torch.stack([x["gate"] for x in xs])
    bias = xs[0]["pos_bias"]
    state_x = torch.empty(B, 1, D, dtype=torch.bfloat16, device=DEV)
    state_g = torch.empty(B, 1, D, dtype=torch.bfloat16, device=DEV)
    c8 = torch.zeros(B, S, D - r, dtype=torch.uint8, device=DEV)
    c8s = torch.zeros(B, S, dtype=torch.float32, device=DEV)
    crope = torch.zeros(B, S, r, dtype=torch.bfloat16, device=DEV)
    kv_d, gate_d = kv.to(DEV), gate.to(DEV)
    for P in range(S):
        csa.compress_append(kv_d[:, P].contiguous(), gate_d[:, P].contiguous(), bias.to(DEV), state_x, state_g, P,
                            1, r, wl.theta_cmp, wl.theta_tok, c8=c8, c8_scale=c8s, c_rope=crope)
    torch.cuda.synchronize()
    for b in range(B):
        rc, rs = oracle.fp8_entry_rows(kv[b, :, :D - r].float().numpy())
        assert np.array_equal(c8s[b].cpu().numpy(), rs), "scales"
        assert np.array_equal(c8[b].cpu().numpy(), rc), "codes"
        Cr, _ = oracle.compress(kv[b], gate[b], bias, 1, 1, r, wl.theta_cmp, wl.theta_tok)
        bf16_rel_close(crope[b].float().cpu(), Cr[:, D - r:], "rope channels")
    assert c8s[0, 0].item() == 1.0


def test_compress_append_fp8_cache():
    """FP8 entry cache of the CSA compressor (m = 4, L = 8): rope channels in bf16; scales equal the
    oracle's amax/448 to binary32 rounding of the pooled values; codes equal the oracle's encoding of
    the oracle's pooled value over the GPU's scale, apart from counted near-boundary quotients."""
    wl = WORKLOADS[1].with_(m=4, L=8)
    S, B, D, r = 41, 2, wl.D, wl.r
    _, _, _, _, cache, refs = _append_history(wl, B, S, fp8=True)
    T = S // wl.m
    for b in range(B):
        Cr = refs[b][0][:T]
        nope, rope = Cr[:, : D - r], Cr[:, D - r:]
        scale = cache["c8_scale"][b].cpu().numpy()
        _, rs = oracle.fp8_entry_rows(nope)
        np.testing.assert_allclose(scale, rs, rtol=2.0 ** -20, atol=0)
        _fp8_codes_match(cache["c8"][b].cpu().numpy(), nope, scale, "codes", max_ties=8)
        bf16_rel_close(cache["c_rope"][b].float().cpu(), rope, "rope channels")


def test_compress_append_feeds_decode():
    """The caches written by the decode step serve the decode attention directly: hca_decode on the
    entry cache and the window ring equals the oracle's decode on the prefill compressor's entries and
    the window rows in position order (the ring order does not matter to the attention)."""
    wl = WORKLOADS[1].with_(m=4, L=8)
    S, B = 300, 2
    _, _, _, win, cache, refs = _append_history(wl, B, S)
    T, W, P = S // wl.m, wl.W, S - 1
    q = torch.randn(B, wl.H, wl.D, generator=torch.Generator().manual_seed(7)).mul_(wl.q_std).to(torch.bfloat16)
    sinks = torch.randn(wl.H, generator=torch.Generator().manual_seed(8))
    o = csa.hca_decode(q.to(DEV), win, sinks.to(DEV), P, wl.r, wl.theta_tok, wl.theta_cmp, C=cache["C"])
    torch.cuda.synchronize()
    Cb = torch.stack([torch.tensor(refs[b][0][:T]) for b in range(B)]).to(torch.bfloat16)
    winb = torch.stack([torch.tensor(refs[b][1][P - W + 1:P + 1]) for b in range(B)]).to(torch.bfloat16)
    ref = oracle.decode_attend(q, winb, np.tile(np.arange(T, dtype=np.int32), (B, 1)), sinks, P, wl.r, wl.theta_tok,
                               wl.theta_cmp, C=Cb)
    check_close(o.cpu(), ref, O_MAX_ABS, O_MEAN_ABS, what="o")


# ---- 9. grouped output projection --------------------------------------------------------------------

def _proj_close(got, ref, what):
    got = got.float().cpu().double().numpy()
    ref = np.asarray(ref)
    rms = float(np.sqrt((ref ** 2).mean()))
    bad = np.abs(got - ref) > 2.0 ** -8 * np.abs(ref) + 2e-3 * rms
    assert not bad.any(), f"{what}: {int(bad.sum())} values beyond bf16 rounding (rms {rms:.3g})"


@pytest.mark.parametrize("S", [300, 130])
def test_out_proj(S):
    """V4-Flash shapes (8 groups of 8 heads x 512 -> 1024 each -> 4096); S=130 leaves a ragged row tile."""
    from workloads import proj_inputs
    wl = WORKLOADS[7].with_(S=S)
    g = proj_inputs(wl, device=DEV)
    z, out = csa.out_proj(g["o"], g["wa"], g["wb"])
    torch.cuda.synchronize()
    h = host(g)
    zr, outr = oracle.out_proj(h["o"], h["wa"], h["wb"])
    _proj_close(z, zr, "z")
    _proj_close(out, outr, "out")


def test_out_proj_full_size_sampled():
    """S=8192 as the benchmark runs it, checked on sampled rows (rows are independent)."""
    from workloads import proj_inputs
    wl = WORKLOADS[7]
    g = proj_inputs(wl, device=DEV)
    z, out = csa.out_proj(g["o"], g["wa"], g["wb"])
    torch.cuda.synchronize()
    rows = sample_rows(wl.S, 24, 17, must=[0, 127, 128, wl.S - 1])
    zr, outr = oracle.out_proj(g["o"][rows].cpu(), g["wa"].cpu(), g["wb"].cpu())
    _proj_close(z[rows], zr, "z")
    _proj_close(out[rows], outr, "out")


# ---- 10. empty inputs --------------------------------------------------------------------------------

def test_empty_inputs():
    """Zero tokens or zero sequences: every call succeeds and returns empty outputs."""
    from workloads import proj_inputs
    wl = WORKLOADS[1].with_(S=0)
    g = prefill_inputs(wl, device=DEV)
    o, C, kv_rot, idx = csa.csa_forward(g["q"], g["kv"], g["gate"], g["pos_bias"], g["qI"], g["kI"], g["w"],
                                        g["sinks"], wl.m, wl.L, wl.topk, wl.W, wl.r, wl.theta_tok, wl.theta_cmp)
    assert o.shape == (0, wl.H, wl.D) and C.shape[0] == 0 and idx.shape[0] == 0
    h = prefill_inputs(WORKLOADS[2].with_(S=0), device=DEV)
    o, C, _ = csa.hca_forward(h["q"], h["kv"], h["gate"], h["pos_bias"], h["sinks"], 128, 128, wl.W, wl.r,
                              wl.theta_tok, wl.theta_cmp)
    assert o.shape == (0, wl.H, wl.D)
    dw = WORKLOADS[3].with_(ctx=4096)
    y = decode_inputs(dw, device=DEV, batch=0)
    o, idx = csa.decode(y["q"], y["qI"], y["w"], y["kI"], y["win"], y["sinks"], dw.ctx - 1, dw.topk, dw.r,
                        dw.theta_tok, dw.theta_cmp, C=y["C"])
    assert o.shape == (0, dw.H, dw.D) and idx.shape == (0, dw.topk)
    o = csa.hca_decode(y["q"], y["win"], y["sinks"], dw.ctx - 1, dw.r, dw.theta_tok, dw.theta_cmp, C=y["C"])
    assert o.shape == (0, dw.H, dw.D)
    p = proj_inputs(WORKLOADS[7].with_(S=0), device=DEV)
    z, out = csa.out_proj(p["o"], p["wa"], p["wb"])
    assert z.shape == (0, 8 * 1024) and out.shape == (0, 4096)
    torch.cuda.synchronize()
