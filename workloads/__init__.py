"""Seeded synthetic workloads for the CSA / HCA attention forward.

This module only draws random inputs and describes workload shapes. It contains none of the
method's arithmetic: no pooling, no RoPE, no scoring, no attention. Both the CUDA path's tests and
benchmarks and the CPU oracle's tests take their inputs from here.

Shapes follow the DeepSeek-V4-Flash attention layer (llm-atlas model card "DeepSeek-V4-Flash",
table "config.json full fields": head_dim 512, 64 heads, one KV head, qk_rope_head_dim 64,
index_n_heads 64, index_head_dim 128, index_topk 512, sliding_window 128, rope_theta 10000,
compress_rope_theta 160000) and the CSA / HCA compression rates m=4 / m'=128 (Hugging Face
Transformers docs "DeepSeek-V4", section "Hybrid attention").

Every tensor is drawn by torch's counter-based Philox (CUDA) or Mersenne (CPU) generator seeded by
(workload seed, tensor id), then rounded to bf16 by round-to-nearest-even where the layout is bf16.
The same seed on the same device gives the same bits on every run.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, Optional

import torch

__all__ = ["Workload", "WORKLOADS", "prefill_inputs", "attend_inputs", "decode_inputs", "proj_inputs", "tensor_gen"]


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    kind: str                 # "csa_prefill" | "hca_prefill" | "csa_decode" | "hca_decode" | "compress_append"
    S: int = 0                # prefill tokens
    H: int = 64
    D: int = 512
    m: int = 4                # compression stride
    L: int = 8                # pooling window length (2m for CSA, m for HCA)
    HI: int = 64              # index heads
    dI: int = 128             # index head dim
    topk: int = 512
    W: int = 128              # sliding window
    r: int = 64               # rope dims
    theta_tok: float = 10000.0
    theta_cmp: float = 160000.0
    q_std: float = 1.0 / math.sqrt(512.0)
    seed: int = 0
    # decode only
    B: int = 0
    ctx: int = 0              # tokens of history per sequence
    cache: str = "bf16"       # "bf16" | "fp8"
    index_fmt: str = "bf16"   # indexer operands q^I, k^I: "bf16" | "fp4" (MXFP4)
    # grouped output projection (o_groups, o_lora_rank, hidden_size of the V4-Flash config)
    o_groups: int = 8
    o_rank: int = 1024
    hidden: int = 4096

    @property
    def T(self) -> int:
        return (self.ctx if self.kind in ("csa_decode", "hca_decode", "compress_append") else self.S) // self.m

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five workloads: a tiny CSA layer, the V4-Flash CSA prefill layer, the V4-Flash HCA prefill
# layer, CSA decode at 128K context and CSA decode at 1M context with an FP8 entry cache.
WORKLOADS: Dict[int, Workload] = {
    0: Workload("tiny_csa_prefill_s1024", "csa_prefill", S=1024, H=8, D=128, m=4, L=8, HI=4, dI=64,
                topk=16, W=128, r=32, theta_tok=10000.0, theta_cmp=10000.0, q_std=1.0, seed=0),
    1: Workload("v4flash_csa_prefill_s8192", "csa_prefill", S=8192, seed=1),
    2: Workload("v4flash_hca_prefill_s65536", "hca_prefill", S=65536, m=128, L=128, HI=0, dI=0,
                topk=0, seed=2),
    3: Workload("csa_decode_b64_ctx128k", "csa_decode", B=64, ctx=131072, topk=1024, seed=3),
    4: Workload("csa_decode_b8_ctx1m_fp8", "csa_decode", B=8, ctx=1048576, topk=512, cache="fp8", seed=4),
    # beyond the five: HCA decode at 1M context (m' = 128: 8192 pooled entries per sequence, all attended)
    5: Workload("hca_decode_b8_ctx1m", "hca_decode", B=8, ctx=1048576, m=128, L=128, topk=0, seed=5),
    # the CSA compressor's decode step for 64 sequences at 128K context (m = 4 appends close one entry)
    6: Workload("csa_append_b64_ctx128k", "compress_append", B=64, ctx=131072, m=4, L=8, topk=0, seed=6),
    # the grouped output projection after the V4-Flash attention, S=8192
    7: Workload("v4flash_out_proj_s8192", "out_proj", S=8192, seed=7),
    # CSA decode at 128K context with the FP4 (MXFP4) lightning indexer: k^I cached as MXFP4
    8: Workload("csa_decode_b64_ctx128k_fp4idx", "csa_decode", B=64, ctx=131072, topk=1024, seed=3, index_fmt="fp4"),
}


def tensor_gen(seed: int, tensor_id: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) * 1009 + int(tensor_id))
    return g


def _normal(shape, std, seed, tid, device, dtype=torch.bfloat16):
    g = tensor_gen(seed, tid, device)
    x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(dtype)


def _uniform(shape, seed, tid, device):
    g = tensor_gen(seed, tid, device)
    return torch.rand(shape, generator=g, device=device, dtype=torch.float32)


# tensor ids (stable: changing one changes that tensor only)
_Q, _KV, _GATE, _BIAS, _QI, _KI, _WI, _SINK, _C, _KVROT, _WIN, _O, _WA, _WB = range(14)


def prefill_inputs(wl: Workload, device="cpu", need_index: Optional[bool] = None,
                   need_q: bool = True) -> Dict[str, torch.Tensor]:
    """q [S,H,D] bf16, kv/gate [S,D] bf16, pos_bias [L] f32, sinks [H] f32 and, for CSA,
    q^I [S,HI,dI] bf16, k^I [T,dI] bf16 (one index key per entry), w [S,HI] f32."""
    S, H, D, T = wl.S, wl.H, wl.D, wl.T
    out = {
        "kv": _normal((S, D), 1.0, wl.seed, _KV, device),
        "gate": _normal((S, D), 1.0, wl.seed, _GATE, device),
        "pos_bias": _normal((wl.L,), 0.02, wl.seed, _BIAS, device, torch.float32),
        "sinks": _normal((H,), 1.0, wl.seed, _SINK, device, torch.float32),
    }
    if need_q:
        out["q"] = _normal((S, H, D), wl.q_std, wl.seed, _Q, device)
    if need_index is None:
        need_index = wl.kind == "csa_prefill"
    if need_index:
        out["qI"] = _normal((S, wl.HI, wl.dI), 1.0, wl.seed, _QI, device)
        out["kI"] = _normal((T, wl.dI), 1.0, wl.seed, _KI, device)
        out["w"] = _uniform((S, wl.HI), wl.seed, _WI, device)
    return out


def attend_inputs(wl: Workload, device="cpu") -> Dict[str, torch.Tensor]:
    """Stand-alone attention inputs: post-RoPE entry rows C [T,D] and window rows kv_rot [S,D]
    drawn directly (as a cache would hold them), so attention can be checked without the compressor."""
    return {
        "C": _normal((wl.T, wl.D), 1.0, wl.seed, _C, device),
        "kv_rot": _normal((wl.S, wl.D), 1.0, wl.seed, _KVROT, device),
    }


def decode_inputs(wl: Workload, device="cpu", batch: Optional[int] = None) -> Dict[str, torch.Tensor]:
    """One query per sequence against post-RoPE caches.

    q [B,H,D] bf16 (un-rotated), q^I [B,HI,dI] bf16, w [B,HI] f32, k^I [B,T,dI] bf16,
    window rows win [B,W,D] bf16 (positions P-W+1..P), sinks [H] f32 and either
    C [B,T,D] bf16 or the FP8 triplet c8 [B,T,D-r] uint8 (E4M3 codes), scale [B,T] f32,
    rope [B,T,r] bf16."""
    B = wl.B if batch is None else batch
    T, D, r = wl.T, wl.D, wl.r
    out = {
        "q": _normal((B, wl.H, D), wl.q_std, wl.seed, _Q, device),
        "qI": _normal((B, wl.HI, wl.dI), 1.0, wl.seed, _QI, device),
        "w": _uniform((B, wl.HI), wl.seed, _WI, device),
        "kI": _normal((B, T, wl.dI), 1.0, wl.seed, _KI, device),
        "win": _normal((B, wl.W, D), 1.0, wl.seed, _WIN, device),
        "sinks": _normal((wl.H,), 1.0, wl.seed, _SINK, device, torch.float32),
    }
    if wl.cache == "fp8":
        x = _normal((B, T, D), 1.0, wl.seed, _C, device, torch.float32)
        nope = x[..., : D - r]
        amax = nope.abs().amax(dim=-1)
        scale = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))
        codes = (nope / scale.unsqueeze(-1)).clamp_(-448.0, 448.0).to(torch.float8_e4m3fn)
        out["c8"] = codes.view(torch.uint8).contiguous()
        out["scale"] = scale.contiguous()
        out["rope"] = x[..., D - r:].to(torch.bfloat16).contiguous()
        del x, nope
    else:
        out["C"] = _normal((B, T, D), 1.0, wl.seed, _C, device)
    return out


def proj_inputs(wl: Workload, device="cpu") -> Dict[str, torch.Tensor]:
    """Grouped output projection inputs: the attention output o [S, H*D] bf16 ~ N(0, 0.25^2) and
    synthetic weights wa [G, R, (H/G)*D], wb [hidden, G*R] bf16 ~ N(0, 1/fan_in)."""
    G, R, hid = wl.o_groups, wl.o_rank, wl.hidden
    K = wl.H // G * wl.D
    return {
        "o": _normal((wl.S, wl.H * wl.D), 0.25, wl.seed, _O, device),
        "wa": _normal((G, R, K), 1.0 / math.sqrt(K), wl.seed, _WA, device),
        "wb": _normal((hid, G * R), 1.0 / math.sqrt(G * R), wl.seed, _WB, device),
    }
