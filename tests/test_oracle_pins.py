"""Pins of the fp64 oracle to facts outside itself (CPU only).

Each test checks the oracle against something it does not share code with: a textbook dense
attention written with complex-number RoPE, closed forms of the pooling, softmax and sink
identities, brute force over subsets, hand-worked small cases, torch's own bf16 / FP8 decoders,
and the worked mask example printed on the Hugging Face Transformers "DeepSeek-V4" page
(section "Attention mask layout"). Each is chosen so that a plausible slip in the oracle
(a dropped bias, a shifted window, a wrong rotation sign, ReLU after the head sum, a missing sink,
a top-k tie broken the wrong way) fails at least one of them.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from workloads import WORKLOADS, prefill_inputs, attend_inputs, decode_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---- independent helpers (complex-number RoPE, textbook softmax attention) -----------------------

def rope_complex(x, r, pos, theta):
    """RoPE written as complex multiplication of interleaved pairs: (x0 + i x1) * e^{i pos f_p}."""
    x = np.array(x, np.float64, copy=True)
    D = x.shape[-1]
    z = x[..., D - r::2] + 1j * x[..., D - r + 1::2]
    f = theta ** (-np.arange(r // 2) * 2.0 / r)
    z = z * np.exp(1j * np.multiply.outer(np.asarray(pos, np.float64), f))
    x[..., D - r::2] = z.real
    x[..., D - r + 1::2] = z.imag
    return x


def bf16(x):
    return torch.tensor(np.asarray(x, np.float32)).to(torch.bfloat16)


def dense_causal_reference(q, k, sinks, r, theta, scale):
    """Textbook causal MQA with K = V = RoPE(k), sink in the denominator, output de-rotated at -t."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    S, H, D = q.shape
    pos = np.arange(S)
    kr = rope_complex(k, r, pos, theta)
    out = np.zeros((S, H, D))
    for t in range(S):
        qt = rope_complex(q[t], r, np.full(H, t), theta)
        logits = scale * qt @ kr[: t + 1].T                       # [H, t+1]
        mx = np.maximum(logits.max(1), sinks)
        e = np.exp(logits - mx[:, None])
        den = e.sum(1) + np.exp(sinks - mx)
        u = (e / den[:, None]) @ kr[: t + 1]
        out[t] = rope_complex(u, r, np.full(H, -t), theta)
    return out


def f64(t):
    return t.float().double().numpy()


# ---- P-dense: m=1 compression with a full top-k is dense causal attention ------------------------

@pytest.mark.parametrize("mode", ["hca", "csa"])
def test_dense_equivalence(mode):
    S, H, D, r, theta = 24, 3, 16, 8, 10000.0
    g = torch.Generator().manual_seed(11)
    q = torch.randn(S, H, D, generator=g).to(torch.bfloat16)
    kv = torch.randn(S, D, generator=g).to(torch.bfloat16)
    gate = torch.randn(S, D, generator=g).to(torch.bfloat16)
    sinks = torch.randn(H, generator=g)
    scale = 0.3
    if mode == "hca":
        # HCA with m'=1: each entry pools one token (a 1-element softmax is 1).
        C, kvr = oracle.compress(kv, gate, torch.zeros(1), m=1, L=1, r=r, theta_cmp=theta, theta_tok=theta)
        idx = None
    else:
        # CSA with m=1: the previous-token offset carries bias -inf, so entry w = kv[w];
        # top-k with k >= S keeps every visible entry.
        C, kvr = oracle.compress(kv, gate, torch.tensor([-math.inf, 0.0]), m=1, L=2, r=r,
                                 theta_cmp=theta, theta_tok=theta)
        qI = torch.randn(S, 2, 4, generator=g).to(torch.bfloat16)
        kI = torch.randn(S, 4, generator=g).to(torch.bfloat16)
        w = torch.rand(S, 2, generator=g)
        idx, _ = oracle.index_topk(qI, kI, w, m=1, k=S + 3)
    out = oracle.attend(q, C, kvr, idx, sinks, m=1, W=0, r=r, theta_tok=theta, theta_cmp=theta, scale=scale)
    ref = dense_causal_reference(f64(q), f64(kv), sinks.double().numpy(), r, theta, scale)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)


def test_window_only_is_banded_dense():
    """No entries at all (k=0 slots): the window branch alone is banded causal attention."""
    S, H, D, r, theta, W = 20, 2, 8, 4, 500.0, 5
    g = torch.Generator().manual_seed(5)
    q = torch.randn(S, H, D, generator=g).to(torch.bfloat16)
    kv = torch.randn(S, D, generator=g).to(torch.bfloat16)
    sinks = torch.randn(H, generator=g)
    _, kvr = oracle.compress(kv, kv, torch.zeros(1), m=1, L=1, r=r, theta_cmp=theta, theta_tok=theta,
                             want_C=False)
    C = np.zeros((1, D))
    idx = np.full((S, 1), -1, np.int32)
    out = oracle.attend(q, C, kvr, idx, sinks, m=1, W=W, r=r, theta_tok=theta, theta_cmp=theta)
    qn, kn = f64(q), f64(kv)
    kr = rope_complex(kn, r, np.arange(S), theta)
    for t in range(S):
        lo = max(0, t - W + 1)
        qt = rope_complex(qn[t], r, np.full(H, t), theta)
        lg = qt @ kr[lo: t + 1].T / math.sqrt(D)
        e = np.exp(lg)
        p = e / (e.sum(1) + np.exp(sinks.double().numpy()))[:, None]
        ref = rope_complex(p @ kr[lo: t + 1], r, np.full(H, -t), theta)
        np.testing.assert_allclose(out[t], ref, atol=1e-12)


# ---- P-sink ----------------------------------------------------------------------------------------

def test_sink_closed_form_identical_keys():
    """All keys equal v (r=0, no rotation): o = n e^l / (e^z + n e^l) * v for every head."""
    S, H, D = 9, 4, 6
    v = np.linspace(-1, 1, D)
    kv = bf16(np.tile(v, (S, 1)))
    q = bf16(np.random.default_rng(0).normal(size=(S, H, D)))
    sinks = torch.tensor([-math.inf, -2.0, 0.5, 3.0])
    _, kvr = oracle.compress(kv, kv, torch.zeros(1), m=1, L=1, r=0, theta_cmp=1.0, theta_tok=1.0, want_C=False)
    W = 4
    idx = np.full((S, 1), -1, np.int32)
    out = oracle.attend(q, np.zeros((1, D)), kvr, idx, sinks, m=1, W=W, r=0, theta_tok=1.0, theta_cmp=1.0, scale=0.7)
    vv = f64(kv)[0]
    qn = f64(q)
    for t in range(S):
        n = min(W, t + 1)
        for h in range(H):
            l = 0.7 * float(qn[t, h] @ vv)
            z = float(sinks[h])
            frac = n * math.exp(l) / (math.exp(z) + n * math.exp(l))
            np.testing.assert_allclose(out[t, h], frac * vv, atol=1e-13)


def test_sink_limits():
    S, H, D, r = 12, 2, 8, 4
    g = torch.Generator().manual_seed(3)
    q = torch.randn(S, H, D, generator=g).to(torch.bfloat16)
    kv = torch.randn(S, D, generator=g).to(torch.bfloat16)
    C, kvr = oracle.compress(kv, kv, torch.zeros(1), m=1, L=1, r=r, theta_cmp=100.0, theta_tok=100.0)
    big = oracle.attend(q, C, kvr, None, torch.tensor([200.0, 200.0]), m=1, W=3, r=r, theta_tok=100.0, theta_cmp=100.0)
    assert np.abs(big).max() < 1e-60
    none = oracle.attend(q, C, kvr, None, torch.tensor([-math.inf, -math.inf]), m=1, W=0, r=r,
                         theta_tok=100.0, theta_cmp=100.0, scale=0.25)
    # without a sink the weights of a single visible key are 1: row 0 returns that key exactly
    np.testing.assert_allclose(none[0, 0], rope_complex(rope_complex(f64(kv)[0], r, 0, 100.0), r, 0, 100.0), atol=1e-13)
    ref = dense_causal_reference(f64(q), f64(kv), np.array([-np.inf, -np.inf]), r, 100.0, 0.25)
    np.testing.assert_allclose(none, ref, atol=1e-12)


# ---- P-pool: closed forms of the softmax-gated pooling ---------------------------------------------

def test_pool_constant_kv():
    S, D, m, L = 26, 5, 4, 8
    rng = np.random.default_rng(1)
    kv = bf16(np.full((S, D), 1.375))
    gate = bf16(rng.normal(size=(S, D)))
    b = torch.tensor(rng.normal(size=L), dtype=torch.float32)
    C, _ = oracle.compress(kv, gate, b, m=m, L=L, r=0, theta_cmp=1.0, theta_tok=1.0, want_kv_rot=False)
    assert C.shape == (S // m, D)            # the trailing partial block makes no entry
    np.testing.assert_allclose(C, 1.375, atol=1e-15)


@pytest.mark.parametrize("m,L", [(4, 8), (8, 8), (3, 6)])
def test_pool_constant_gate_is_window_mean(m, L):
    S, D = 5 * m + 2, 3
    kv = bf16(np.random.default_rng(2).normal(size=(S, D)))
    gate = bf16(np.full((S, D), -0.5))
    C, _ = oracle.compress(kv, gate, torch.zeros(L), m=m, L=L, r=0, theta_cmp=1.0, theta_tok=1.0, want_kv_rot=False)
    kvn = f64(kv)
    for w in range(S // m):
        lo, hi = max(0, (w + 1) * m - L), (w + 1) * m
        np.testing.assert_allclose(C[w], kvn[lo:hi].mean(0), atol=1e-14)
    if L == 2 * m:   # CSA: entry 0 pools only its own m tokens, entry 1 pools 2m
        np.testing.assert_allclose(C[0], kvn[:m].mean(0), atol=1e-14)
        np.testing.assert_allclose(C[1], kvn[: 2 * m].mean(0), atol=1e-14)


def test_pool_zero_gate_weights_are_softmax_of_bias():
    S, D, m, L = 16, 2, 4, 8
    kv = bf16(np.random.default_rng(3).normal(size=(S, D)))
    b = np.array([0.3, -1.0, 2.0, 0.0, 0.5, -0.25, 1.5, -2.0])
    C, _ = oracle.compress(kv, bf16(np.zeros((S, D))), torch.tensor(b, dtype=torch.float32), m=m, L=L, r=0,
                           theta_cmp=1.0, theta_tok=1.0, want_kv_rot=False)
    b32 = np.float32(b).astype(np.float64)
    kvn = f64(kv)
    full = np.exp(b32) / np.exp(b32).sum()
    for w in range(1, S // m):
        np.testing.assert_allclose(C[w], full @ kvn[(w - 1) * m:(w + 1) * m], atol=1e-14)
    half = np.exp(b32[m:]) / np.exp(b32[m:]).sum()     # entry 0: offsets m..2m-1 only
    np.testing.assert_allclose(C[0], half @ kvn[:m], atol=1e-14)


def test_pool_entry_rotation_position():
    """Entries are rotated at p_w = w*m with theta_cmp; kv_rot[j] at j with theta_tok."""
    S, D, m, L, r = 16, 8, 4, 8, 4
    rng = np.random.default_rng(4)
    kv, gate = bf16(rng.normal(size=(S, D))), bf16(rng.normal(size=(S, D)))
    b = torch.tensor(rng.normal(size=L), dtype=torch.float32)
    C0, _ = oracle.compress(kv, gate, b, m=m, L=L, r=0, theta_cmp=1.0, theta_tok=1.0)
    C, kvr = oracle.compress(kv, gate, b, m=m, L=L, r=r, theta_cmp=160000.0, theta_tok=10000.0)
    np.testing.assert_allclose(C, rope_complex(C0, r, np.arange(S // m) * m, 160000.0), atol=1e-13)
    np.testing.assert_allclose(kvr, rope_complex(f64(kv), r, np.arange(S), 10000.0), atol=1e-13)


# ---- P-rope ------------------------------------------------------------------------------------------

def test_rope_matches_complex_form_and_inverts():
    rng = np.random.default_rng(5)
    x = rng.normal(size=12)
    for pos, theta in [(0, 1e4), (7, 1e4), (131071, 1.6e5), (1048575, 1e4)]:
        y = oracle.rope(x, 8, pos, theta)
        np.testing.assert_allclose(y, rope_complex(x, 8, pos, theta), atol=1e-9)
        assert abs(np.linalg.norm(y) - np.linalg.norm(x)) < 1e-12
        np.testing.assert_allclose(oracle.rope(y, 8, -pos, theta), x, atol=1e-9)
        np.testing.assert_array_equal(y[:4], x[:4])   # only the last r channels rotate


def test_single_entry_is_relative_rotation():
    """One selected entry, no window: o_rope = (1 - p_sink) R(p_s - t) v_rope."""
    S, D, r, m = 12, 6, 4, 1
    rng = np.random.default_rng(6)
    kv = bf16(rng.normal(size=(S, D)))
    C, kvr = oracle.compress(kv, kv, torch.tensor([-math.inf, 0.0]), m=m, L=2, r=r, theta_cmp=40.0, theta_tok=9.0)
    q = bf16(rng.normal(size=(S, 1, D)))
    s_sel = 3
    idx = np.full((S, 1), -1, np.int32)
    idx[s_sel:, 0] = s_sel
    sinks = torch.tensor([0.2])
    out = oracle.attend(q, C, kvr, idx, sinks, m=m, W=0, r=r, theta_tok=9.0, theta_cmp=40.0, scale=0.5)
    v = f64(kv)[s_sel]
    for t in range(s_sel, S):
        qt = rope_complex(f64(q)[t, 0], r, t, 40.0)
        l = 0.5 * float(qt @ rope_complex(v, r, s_sel, 40.0))
        p = math.exp(l) / (math.exp(l) + math.exp(0.2))
        np.testing.assert_allclose(out[t, 0], p * rope_complex(v, r, s_sel - t, 40.0), atol=1e-13)


def test_window_branch_shift_invariance():
    """One theta, window only: moving the query and every window row by the same offset leaves
    the output unchanged (each row contributes as a function of its distance to the query)."""
    B, H, D, r, W, theta = 1, 3, 8, 4, 6, 1e4
    rng = np.random.default_rng(7)
    v = rng.normal(size=(W, D))
    q = bf16(rng.normal(size=(B, H, D)))
    sinks = torch.tensor(rng.normal(size=H), dtype=torch.float32)
    outs = []
    for P in (20, 20 + 1000, 20 + 77777):
        win = rope_complex(v, r, np.arange(P - W + 1, P + 1), theta)
        winb = bf16(win)[None]
        # the bf16 rounding of the rotated rows differs per P; compare against a tolerance that
        # covers it, and exactly against an un-rounded twin below
        outs.append(oracle.decode_attend(q, winb, np.full((B, 1), -1, np.int32), sinks, P, r, theta, theta,
                                         C=bf16(np.zeros((B, 1, D)))))
    for o in outs[1:]:
        np.testing.assert_allclose(o, outs[0], atol=2e-2)
    # un-rounded: prefill rows built in double, compared across two shifted windows exactly
    S = 40
    kv = rng.normal(size=(S, D))
    qq = rng.normal(size=(S, H, D))
    kvb, qb = bf16(kv), bf16(qq)
    _, kvr = oracle.compress(kvb, kvb, torch.zeros(1), m=1, L=1, r=r, theta_cmp=theta, theta_tok=theta, want_C=False)
    idx = np.full((S, 1), -1, np.int32)
    o = oracle.attend(qb, np.zeros((1, D)), kvr, idx, sinks, m=1, W=W, r=r, theta_tok=theta, theta_cmp=theta)
    base = f64(kvb)
    for t in (10, 25):
        rel = rope_complex(base[t - W + 1: t + 1], r, np.arange(-W + 1, 1), theta)   # positions relative to t
        lg = rope_complex(f64(qb)[t], r, np.zeros(H), theta) @ rel.T / math.sqrt(D)
        e = np.exp(lg)
        p = e / (e.sum(1) + np.exp(sinks.double().numpy()))[:, None]
        np.testing.assert_allclose(o[t], p @ rel, atol=1e-12)


def test_dual_theta_branches_rotate_with_their_own_theta():
    """theta_tok != theta_cmp: each branch de-rotates with its own theta (checked by q=0, so all
    logits are 0 and every key weighs 1/(e^z + n))."""
    S, D, r, m, L, W = 16, 8, 4, 2, 4, 3
    rng = np.random.default_rng(8)
    kv, gate = bf16(rng.normal(size=(S, D))), bf16(rng.normal(size=(S, D)))
    b = torch.tensor(rng.normal(size=L), dtype=torch.float32)
    tt, tc = 10000.0, 160000.0
    C, kvr = oracle.compress(kv, gate, b, m=m, L=L, r=r, theta_cmp=tc, theta_tok=tt)
    C0, _ = oracle.compress(kv, gate, b, m=m, L=L, r=0, theta_cmp=1.0, theta_tok=1.0)
    q = bf16(np.zeros((S, 1, D)))
    k = 2
    idx = np.full((S, k), -1, np.int32)
    for t in range(S):
        vis = (t + 1) // m
        sel = list(range(max(0, vis - k), vis))
        idx[t, : len(sel)] = sel
    z = -0.3
    out = oracle.attend(q, C, kvr, idx, torch.tensor([z]), m=m, W=W, r=r, theta_tok=tt, theta_cmp=tc)
    kvn = f64(kv)
    for t in range(S):
        win = list(range(max(0, t - W + 1), t + 1))
        sel = [s for s in idx[t] if s >= 0]
        n = len(win) + len(sel)
        p = 1.0 / (math.exp(z) + n)
        ref = np.zeros(D)
        for j in win:
            ref += p * rope_complex(kvn[j], r, j - t, tt)
        for s in sel:
            ref += p * rope_complex(C0[s], r, s * m - t, tc)
        np.testing.assert_allclose(out[t, 0], ref, atol=1e-13)


# ---- P-causal and the page's worked mask example ----------------------------------------------------

def test_mask_example_from_page():
    spec = json.load(open(os.path.join(GOLDEN, "mask_16tok.json")))
    cfg = spec["config"]
    S, m_hca, m_csa, k = cfg["S"], cfg["hca_m"], cfg["csa_m"], cfg["index_topk"]
    T_hca = S // m_hca
    for e, t_first in spec["statements"]["hca_entry_first_visible_query"].items():
        e = int(e)
        assert all(oracle.visible(t, m_hca, T_hca) <= e for t in range(t_first))
        assert all(oracle.visible(t, m_hca, T_hca) > e for t in range(t_first, S))
    for e, (lo, hi) in spec["statements"]["hca_entry_token_span"].items():
        # entry e of HCA pools exactly tokens lo..hi: a kv that is 1 there and 0 elsewhere pools to 1
        kv = np.zeros((S, 1)); kv[lo: hi + 1] = 1.0
        C, _ = oracle.compress(bf16(kv), bf16(np.zeros((S, 1))), torch.zeros(m_hca), m=m_hca, L=m_hca, r=0,
                               theta_cmp=1.0, theta_tok=1.0, want_kv_rot=False)
        assert C[int(e), 0] == 1.0 and all(C[j, 0] == 0.0 for j in range(T_hca) if j != int(e))
    # CSA: queries t < m-1 receive only -1 sentinels; later queries fill min(k, vis) slots
    g = torch.Generator().manual_seed(0)
    qI, kI, w = torch.randn(S, 2, 4, generator=g).to(torch.bfloat16), torch.randn(S // m_csa, 4, generator=g).to(torch.bfloat16), torch.rand(S, 2, generator=g)
    idx, _ = oracle.index_topk(qI, kI, w, m=m_csa, k=k)
    for t in range(S):
        vis = (t + 1) // m_csa
        if t < m_csa - 1:
            assert (idx[t] == -1).all()
        sel = idx[t][idx[t] >= 0]
        assert len(sel) == min(k, vis) and (sel < vis).all() and len(set(sel.tolist())) == len(sel)
        assert ((idx[t] == -1).any()) == (vis < k)


def test_window_mask_from_page():
    """Sliding mask of the 16-token example (window 8): key j is in the window of i iff i-8 < j <= i.
    Probed with one-hot value rows and q = 0 so each window key weighs the same."""
    S, W = 16, 8
    kv = np.eye(S)
    q = bf16(np.zeros((S, 1, S)))
    kvb = bf16(kv)
    _, kvr = oracle.compress(kvb, kvb, torch.zeros(1), m=1, L=1, r=0, theta_cmp=1.0, theta_tok=1.0, want_C=False)
    out = oracle.attend(q, np.zeros((1, S)), kvr, np.full((S, 1), -1, np.int32), torch.tensor([-math.inf]),
                        m=1, W=W, r=0, theta_tok=1.0, theta_cmp=1.0)
    for i in range(S):
        seen = set(np.nonzero(out[i, 0] > 0)[0].tolist())
        assert seen == {j for j in range(S) if i - W < j <= i}


# ---- P-topk: brute force over subsets -----------------------------------------------------------------

def test_topk_brute_force_with_ties():
    rng = np.random.default_rng(9)
    for trial in range(60):
        n = rng.integers(1, 9)
        k = int(rng.integers(1, 7))
        sc = rng.integers(0, 4, size=n).astype(np.float64)   # many exact ties, zeros included
        got = oracle.topk(sc[None], np.array([n]), k)[0]
        keep = min(k, n)
        best = None
        for sub in itertools.combinations(range(n), keep):    # max score sum, then smallest indices
            key = (-sc[list(sub)].sum(), sub)
            if best is None or key < best:
                best = key
        assert list(got[:keep]) == list(best[1])
        assert (got[keep:] == -1).all()


def test_index_score_relu_per_head_closed_form():
    """Heads x and -x with unit weights give |x.k| (ReLU is per head, before the weighted sum);
    a zero weight removes its head."""
    rng = np.random.default_rng(10)
    S, T, dI, m = 8, 2, 5, 4
    x = rng.normal(size=(S, dI))
    qI = bf16(np.stack([x, -x], axis=1))
    kI = bf16(rng.normal(size=(T, dI)))
    sc = oracle.index_scores(qI, kI, torch.ones(S, 2), m=m)
    qn, kn = f64(qI), f64(kI)
    for t in range(S):
        for s in range(T):
            if s < (t + 1) // m:
                assert abs(sc[t, s] - abs(qn[t, 0] @ kn[s])) < 1e-12
            else:
                assert math.isnan(sc[t, s])
    w = torch.tensor([[1.0, 0.0]] * S)
    sc2 = oracle.index_scores(qI, kI, w, m=m)
    t, s = S - 1, 0
    assert abs(sc2[t, s] - max(0.0, qn[t, 0] @ kn[s])) < 1e-12


# ---- P-8tok: a hand-worked 8-token CSA layer -----------------------------------------------------------

def test_hand_worked_8_tokens():
    """S=8, m=2 (window 4), D=4, r=2, H=1, k=2, W=2, zero gates and bias (pooling = window mean),
    q=0 (every key weighs 1/(1+n) with sink 0), index scores = entry number (top-2 = the two
    newest visible entries). Written out position by position."""
    S, m, L, D, r, k, W = 8, 2, 4, 4, 2, 2, 2
    kv = np.array([[j, 1.0, (-1.0) ** j, 0.5 * j] for j in range(S)])
    kvb = bf16(kv)
    C, kvr = oracle.compress(kvb, bf16(np.zeros((S, D))), torch.zeros(L), m=m, L=L, r=r,
                             theta_cmp=10000.0, theta_tok=10000.0)
    # entries: w=0 mean(kv0,kv1); w=1 mean(kv0..kv3); w=2 mean(kv2..kv5); w=3 mean(kv4..kv7)
    means = [kv[0:2].mean(0), kv[0:4].mean(0), kv[2:6].mean(0), kv[4:8].mean(0)]

    def rot(v, a):   # one pair, frequency 1: angle = position in radians
        c, s = math.cos(a), math.sin(a)
        return np.array([v[0], v[1], v[2] * c - v[3] * s, v[2] * s + v[3] * c])

    for w_, mu in enumerate(means):
        np.testing.assert_allclose(C[w_], rot(mu, 2 * w_), atol=1e-14)
    qI = bf16(np.ones((S, 1, 1)))
    kI = bf16(np.arange(S // m, dtype=np.float64)[:, None])
    idx, _ = oracle.index_topk(qI, kI, torch.ones(S, 1), m=m, k=k)
    expect_idx = [[-1, -1], [0, -1], [0, -1], [0, 1], [0, 1], [1, 2], [1, 2], [2, 3]]
    assert idx.tolist() == expect_idx
    out = oracle.attend(bf16(np.zeros((S, 1, D))), C, kvr, idx, torch.tensor([0.0]), m=m, W=W, r=r,
                        theta_tok=10000.0, theta_cmp=10000.0)
    for t in range(S):
        keys_w = [j for j in (t - 1, t) if j >= 0]
        keys_e = [s for s in expect_idx[t] if s >= 0]
        p = 1.0 / (1.0 + len(keys_w) + len(keys_e))
        ref = sum(p * rot(kv[j], j - t) for j in keys_w) + sum(p * rot(means[s], 2 * s - t) for s in keys_e)
        np.testing.assert_allclose(out[t, 0], ref, atol=1e-14)


# ---- P-decode: decode at P equals row P of prefill ------------------------------------------------------

@pytest.mark.parametrize("cache", ["bf16", "fp8"])
def test_decode_equals_last_prefill_row(cache):
    wl = WORKLOADS[0].with_(S=64, H=3, D=32, r=8, HI=2, dI=8, topk=5, W=6, theta_cmp=160000.0)
    x = prefill_inputs(wl)
    C, kvr = oracle.compress(x["kv"], x["gate"], x["pos_bias"], wl.m, wl.L, wl.r, wl.theta_cmp, wl.theta_tok)
    Cb, kvrb = torch.tensor(C).to(torch.bfloat16), torch.tensor(kvr).to(torch.bfloat16)
    P = wl.S - 1
    T = wl.T
    idx, sc = oracle.index_topk(x["qI"], x["kI"], x["w"], wl.m, wl.topk, rows=[P])
    didx, dsc = oracle.decode_index_topk(x["qI"][P:P + 1], x["w"][P:P + 1], x["kI"][None], wl.topk)
    np.testing.assert_array_equal(didx, idx)
    np.testing.assert_allclose(dsc, sc, atol=0)
    if cache == "fp8":
        nope = Cb.float()[:, : wl.D - wl.r]
        scale = nope.abs().amax(1) / 448.0
        c8 = (nope / scale[:, None]).to(torch.float8_e4m3fn)
        deq = c8.float().double() * scale.double()[:, None]
        Cd = torch.cat([deq, Cb.double()[:, wl.D - wl.r:]], 1)   # exactly what the FP8 cache decodes to
        pre = oracle.attend(x["q"], Cd.numpy(), kvrb, np.broadcast_to(idx, (wl.S, wl.topk)).copy(),
                            x["sinks"], wl.m, wl.W, wl.r, wl.theta_tok, wl.theta_cmp, rows=[P])
        dec = oracle.decode_attend(x["q"][P:P + 1], kvrb[P - wl.W + 1: P + 1][None], idx, x["sinks"], P, wl.r,
                                   wl.theta_tok, wl.theta_cmp, c8=c8.view(torch.uint8)[None], c8_scale=scale[None],
                                   c_rope=Cb[:, wl.D - wl.r:].to(torch.bfloat16)[None])
    else:
        pre = oracle.attend(x["q"], Cb, kvrb, np.broadcast_to(idx, (wl.S, wl.topk)).copy(), x["sinks"], wl.m, wl.W,
                            wl.r, wl.theta_tok, wl.theta_cmp, rows=[P])
        dec = oracle.decode_attend(x["q"][P:P + 1], kvrb[P - wl.W + 1: P + 1][None], idx, x["sinks"], P, wl.r,
                                   wl.theta_tok, wl.theta_cmp, C=Cb[None])
    np.testing.assert_allclose(dec, pre, atol=1e-13)



def test_hca_decode_equals_last_prefill_row():
    """HCA decode reading: decode at P over every cached entry plus the window equals row P of the HCA
    prefill (all entries w < floor((P+1)/m) visible); with no entries it equals the window-only prefill."""
    wl = WORKLOADS[0].with_(S=96, H=3, D=32, r=8, m=16, L=16, W=10, theta_cmp=160000.0)
    x = prefill_inputs(wl, need_index=False)
    C, kvr = oracle.compress(x["kv"], x["gate"], x["pos_bias"], wl.m, wl.L, wl.r, wl.theta_cmp, wl.theta_tok)
    Cb, kvrb = torch.tensor(C).to(torch.bfloat16), torch.tensor(kvr).to(torch.bfloat16)
    P, T = wl.S - 1, wl.T
    assert T == 6
    pre = oracle.attend(x["q"], Cb, kvrb, None, x["sinks"], wl.m, wl.W, wl.r, wl.theta_tok, wl.theta_cmp, rows=[P])
    dec = oracle.decode_attend(x["q"][P:P + 1], kvrb[P - wl.W + 1: P + 1][None], np.arange(T, dtype=np.int32)[None],
                               x["sinks"], P, wl.r, wl.theta_tok, wl.theta_cmp, C=Cb[None])
    np.testing.assert_allclose(dec, pre, atol=1e-13)
    pre0 = oracle.attend(x["q"], Cb[:0], kvrb, None, x["sinks"], 1, wl.W, wl.r, wl.theta_tok, wl.theta_tok, rows=[P])
    dec0 = oracle.decode_attend(x["q"][P:P + 1], kvrb[P - wl.W + 1: P + 1][None], np.zeros((1, 0), np.int32),
                                x["sinks"], P, wl.r, wl.theta_tok, wl.theta_tok, C=Cb[None, :0])
    np.testing.assert_allclose(dec0, pre0, atol=1e-13)

# ---- P-k>=vis: CSA with a covering top-k equals HCA-style dense over visible entries -------------------

def test_csa_full_topk_equals_dense_entries():
    wl = WORKLOADS[0].with_(S=48, H=2, D=16, r=4, HI=2, dI=8, topk=64, W=5)
    x = prefill_inputs(wl)
    y = attend_inputs(wl)
    idx, _ = oracle.index_topk(x["qI"], x["kI"], x["w"], wl.m, wl.topk)
    a = oracle.attend(x["q"], y["C"], y["kv_rot"], idx, x["sinks"], wl.m, wl.W, wl.r, wl.theta_tok, wl.theta_cmp)
    b = oracle.attend(x["q"], y["C"], y["kv_rot"], None, x["sinks"], wl.m, wl.W, wl.r, wl.theta_tok, wl.theta_cmp)
    np.testing.assert_allclose(a, b, atol=1e-14)


# ---- P-fp8 / bf16: decoders against torch's --------------------------------------------------------

def test_fp8_e4m3_all_codes():
    codes = torch.arange(256, dtype=torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).float().double().numpy()
    got = np.array([oracle.e4m3_to_f64(c) for c in range(256)])
    nan = np.isnan(ref)
    assert (np.isnan(got) == nan).all() and nan.sum() == 2 and nan[0x7F] and nan[0xFF]
    np.testing.assert_array_equal(got[~nan], ref[~nan])
    assert got[0x7E] == 448.0 and got[0x01] == 2.0 ** -9 and got[0x08] == 2.0 ** -6


def _e4m3_value(c):
    """E4M3 value of a code from the OCP layout (sign, 4 exponent bits with bias 7, 3 mantissa bits),
    written out here independently of the oracle's decoder."""
    s, e, f = (c >> 7) & 1, (c >> 3) & 15, c & 7
    v = (f / 8.0) * 2.0 ** -6 if e == 0 else (1.0 + f / 8.0) * 2.0 ** (e - 7)
    return -v if s else v


def test_fp8_encode_every_code_round_trips():
    """Every finite code's own value encodes back to that code (both zeros keep their sign)."""
    codes = [c for c in range(256) if c not in (0x7F, 0xFF)]
    vals = np.array([_e4m3_value(c) for c in codes], np.float64)
    vals[codes.index(0x80)] = -0.0
    got = oracle.e4m3_encode(vals.astype(np.float32))
    np.testing.assert_array_equal(got, np.array(codes, np.uint8))


def test_fp8_encode_midpoints_round_to_even_code():
    """Halfway between neighbouring codes the even code wins; just above or below the midpoint the
    nearer code does. Covers the subnormal range, the subnormal/normal seam and every binade."""
    for c in range(0, 0x7E):
        lo, hi = _e4m3_value(c), _e4m3_value(c + 1)
        mid = np.float32((lo + hi) / 2.0)
        assert float(mid) == (lo + hi) / 2.0            # exactly representable in binary32
        even = c if c % 2 == 0 else c + 1
        assert oracle.e4m3_encode(np.array([mid]))[0] == even, hex(c)
        assert oracle.e4m3_encode(np.array([-mid]))[0] == even | 0x80, hex(c)
        up, down = np.nextafter(mid, np.float32(np.inf)), np.nextafter(mid, np.float32(0))
        assert oracle.e4m3_encode(np.array([up]))[0] == c + 1
        assert oracle.e4m3_encode(np.array([down]))[0] == c


def test_fp8_encode_saturates_and_keeps_nan():
    x = np.array([448.0, 449.0, 463.9, 464.0, 1e30, np.inf, -500.0, -np.inf, np.nan, 2.0 ** -11, -2.0 ** -11],
                 np.float32)
    got = oracle.e4m3_encode(x)
    np.testing.assert_array_equal(got, np.array([0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0xFE, 0x7F, 0x00, 0x80],
                                                np.uint8))


def test_fp8_encode_matches_torch_cast_in_range():
    """torch's float8_e4m3fn cast rounds to nearest even; within +-448 it must agree code for code."""
    rng = np.random.default_rng(31)
    x = (rng.standard_normal(200000) * np.exp2(rng.integers(-12, 9, 200000))).astype(np.float32)
    x = x[np.abs(x) <= 448.0]
    ref = torch.tensor(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(oracle.e4m3_encode(x), ref)


def test_fp8_entry_rows_scale_and_codes():
    """Per-row scale amax/448: the largest element becomes code 448, an all-zero row keeps scale 1
    and zero codes, and every decoded element is within half a code step of x / scale."""
    rng = np.random.default_rng(32)
    x = rng.standard_normal((40, 448)).astype(np.float32) * np.float32(3.0)
    x[7] = 0.0
    codes, scale = oracle.fp8_entry_rows(x)
    assert scale[7] == 1.0 and not codes[7].any()
    for i in range(40):
        if i == 7:
            continue
        assert scale[i] == np.float32(np.abs(x[i]).max() / 448.0)
        j = int(np.abs(x[i]).argmax())
        assert codes[i, j] & 0x7F == 0x7E
        q = x[i].astype(np.float64) / float(scale[i])
        dec = np.array([_e4m3_value(int(c)) for c in codes[i]])
        # half the spacing of the binade holding q (3 mantissa bits; subnormal spacing 2^-9)
        half_step = np.exp2(np.maximum(np.floor(np.log2(np.maximum(np.abs(q), 2.0 ** -6))), -6) - 3) / 2
        assert (np.abs(dec - q) <= half_step * (1 + 1e-12)).all()


def test_bf16_decode_matches_torch():
    bits = np.random.default_rng(12).integers(0, 2 ** 16, size=4000, dtype=np.uint16)
    bits = bits[((bits >> 7) & 0xFF) != 0xFF]                                 # finite values
    ref = torch.tensor(bits.view(np.int16)).view(torch.bfloat16).double().numpy()
    got = np.array([oracle.bf16_to_f64(int(b)) for b in bits])
    np.testing.assert_array_equal(got, ref)


# ---- grouped output projection ---------------------------------------------------------------------

def _bf(x):
    return torch.tensor(np.asarray(x, np.float64), dtype=torch.float32).to(torch.bfloat16)


def test_round_bf16_matches_torch():
    x = np.random.default_rng(21).standard_normal(20000).astype(np.float32) * np.float32(3.0)
    got = oracle.round_bf16(x.astype(np.float64))
    ref = torch.tensor(x).to(torch.bfloat16).double().numpy()
    np.testing.assert_array_equal(got, ref)


def test_out_proj_identity_weights():
    """wa[g] = I and wb = I: the projection returns the attention output unchanged."""
    S, G, K = 5, 2, 8
    o = _bf(np.random.default_rng(1).standard_normal((S, G * K)))
    wa = _bf(np.stack([np.eye(K)] * G))
    wb = _bf(np.eye(G * K))
    z, out = oracle.out_proj(o, wa, wb)
    np.testing.assert_array_equal(z, o.double().numpy())
    np.testing.assert_array_equal(out, o.double().numpy())


def test_out_proj_groups_are_separate():
    """The channels of group g depend only on the heads of group g."""
    rng = np.random.default_rng(2)
    S, G, K, R, hid = 4, 3, 6, 5, 7
    o = rng.standard_normal((S, G * K))
    wa, wb = _bf(rng.standard_normal((G, R, K))), _bf(rng.standard_normal((hid, G * R)))
    z, _ = oracle.out_proj(_bf(o), wa, wb)
    o2 = o.copy()
    o2[:, K:2 * K] = 0.0
    z2, _ = oracle.out_proj(_bf(o2), wa, wb)
    np.testing.assert_array_equal(z2[:, R:2 * R], 0.0)
    np.testing.assert_array_equal(z2[:, :R], z[:, :R])
    np.testing.assert_array_equal(z2[:, 2 * R:], z[:, 2 * R:])


def test_out_proj_permutation_weights():
    """A permutation wb reorders the bf16-rounded low-rank channels."""
    rng = np.random.default_rng(3)
    S, G, K, R = 3, 2, 4, 4
    o, wa = _bf(rng.standard_normal((S, G * K))), _bf(rng.standard_normal((G, R, K)))
    perm = rng.permutation(G * R)
    z, out = oracle.out_proj(o, wa, _bf(np.eye(G * R)[perm]))
    np.testing.assert_array_equal(out, oracle.round_bf16(z)[:, perm])


def test_out_proj_brute_force_tiny():
    rng = np.random.default_rng(4)
    S, G, K, R, hid = 2, 2, 3, 2, 3
    o, wa, wb = (_bf(rng.standard_normal(sh)) for sh in [(S, G * K), (G, R, K), (hid, G * R)])
    z, out = oracle.out_proj(o, wa, wb)
    od, wad, wbd = o.double().numpy(), wa.double().numpy(), wb.double().numpy()
    for t in range(S):
        zt = []
        for g in range(G):
            for j in range(R):
                acc = 0.0
                for c in range(K):
                    acc += od[t, g * K + c] * wad[g, j, c]
                zt.append(acc)
        np.testing.assert_allclose(z[t], zt, rtol=1e-15, atol=1e-15)
        zb = oracle.round_bf16(np.array(zt))
        for i in range(hid):
            np.testing.assert_allclose(out[t, i], sum(zb[c] * wbd[i, c] for c in range(G * R)), rtol=1e-14)


# ---- MXFP4 indexer operands (the OCP Microscaling format, which the pages name for the indexer) ----

def test_mxfp4_e2m1_table():
    """The sixteen E2M1 codes decode to the OCP table (sign in bit 3) at scale 2^0 (E8M0 127)."""
    codes = np.array([[c | (c + 1) << 4 for c in range(0, 16, 2)] * 2], np.uint8)   # 16 bytes = 32 values
    vals = oracle.mxfp4_dequantize(codes, np.array([[127]], np.uint8))[0, :16]
    want = [0, 0.5, 1, 1.5, 2, 3, 4, 6, -0.0, -0.5, -1, -1.5, -2, -3, -4, -6]
    assert vals.tolist() == want


def test_mxfp4_rounding_worked_example():
    """amax 7 gives the shared exponent floor(log2 7) - 2 = 0; each value then rounds to the nearest
    E2M1 value, ties to the even code, saturating at 6 (hand-worked)."""
    x = np.zeros((1, 32))
    x[0, :12] = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 7.0, -0.25, -0.3, -2.9, 0.5]
    codes, scales = oracle.mxfp4_quantize(x)
    assert scales.tolist() == [[127]]
    nib = [(b >> (4 * h)) & 15 for b in codes[0].tolist() for h in (0, 1)]
    #          0.25 0.75 1.25 1.75 2.5 3.5 5.0 7.0 -0.25 -0.3  -2.9    0.5
    assert nib[:12] == [0, 2, 2, 4, 4, 6, 6, 7, 0, 8 | 1, 8 | 5, 1]
    assert all(v == 0 for v in nib[12:])


def test_mxfp4_shared_exponent_and_zero_block():
    """The scale exponent follows floor(log2 amax) - 2 across magnitudes; an all-zero block takes
    E8M0 0 and zero codes; the element reaching amax lands in [4, 8) before rounding."""
    for amax, e in [(1.0, 125), (0.75, 124), (4.0, 127), (6.5, 127), (1024.0, 135), (2.0 ** -100, 25)]:
        x = np.zeros((1, 32))
        x[0, 3] = amax
        codes, scales = oracle.mxfp4_quantize(x)
        assert int(scales[0, 0]) == e, (amax, scales)
        assert 4.0 <= amax / 2.0 ** (e - 127) < 8.0
    codes, scales = oracle.mxfp4_quantize(np.zeros((2, 64)))
    assert not codes.any() and not scales.any()


def test_mxfp4_round_trip_on_representable_blocks():
    """Blocks whose values are E2M1 values times 2^(e-127), with at least one magnitude 4 or 6 (so
    the block maximum selects exponent e), quantise back to the same codes and scales."""
    rng = np.random.default_rng(3)
    n = 200
    mag = rng.integers(0, 8, size=(n, 32))
    mag[np.arange(n), rng.integers(0, 32, n)] = rng.choice([6, 7], n)
    sign = rng.integers(0, 2, size=(n, 32)) & (mag > 0)
    e = rng.integers(60, 200, size=n)
    vals = (oracle.E2M1_VALUES[mag] * np.where(sign, -1.0, 1.0)) * np.ldexp(1.0, e - 127)[:, None]
    codes, scales = oracle.mxfp4_quantize(vals)
    assert scales[:, 0].tolist() == e.tolist()
    back = oracle.mxfp4_dequantize(codes, scales)
    assert np.array_equal(back, vals)


def test_fp4_indexer_equals_bf16_indexer_on_fp4_values():
    """With q^I and k^I already MXFP4 values, the FP4 decode indexer selects exactly what the bf16
    indexer selects on the same (exact) values."""
    rng = np.random.default_rng(4)
    B, HI, dI, T, k = 2, 8, 64, 300, 40
    qc, qs = oracle.mxfp4_quantize(rng.standard_normal((B, HI, dI)))
    kc, ks = oracle.mxfp4_quantize(rng.standard_normal((B, T, dI)))
    w = rng.random((B, HI)).astype(np.float32)
    idx4, sc4 = oracle.decode_index_topk_fp4(qc, qs, w, kc, ks, k)
    qv = oracle.mxfp4_dequantize(qc, qs)
    kv = oracle.mxfp4_dequantize(kc, ks)
    # the scores by hand, in fp64, on the dequantised values
    ref = np.einsum("bhd,btd->bht", qv, kv)
    ref = np.einsum("bh,bht->bt", w.astype(np.float64), np.maximum(ref, 0.0))
    assert np.allclose(sc4, ref, rtol=1e-12, atol=1e-12)
    for b in range(B):
        want = np.sort(np.argsort(-ref[b], kind="stable")[:k])
        assert np.array_equal(np.sort(idx4[b][idx4[b] >= 0]), want)
