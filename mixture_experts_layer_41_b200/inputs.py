"""Seeded synthetic workloads for the MoE layer forward.

This module only draws numbers.  It holds none of the layer's arithmetic
(no routing, no capacity, no expert math): it is the one module that both
the CUDA path and the CPU oracle are fed from, so that the two sides read
bit-identical inputs.

Workload shapes follow the pages:
  * Mixtral-style expert MLP, hidden 4096, intermediate 14336, 8 experts,
    top-2 ("moe-architecture" skill page, Operating procedure steps 1-2);
  * Switch-style top-1 routing (same page, step 2 and Decision rules);
  * 256 routed experts with 8 active per token (MoE competition docs,
    "Why MoE Models Are Efficient"), with DeepSeek-V3 sigmoid group routing
    (Edge0 "MoE Spec and Routing", RouterKind / group_select_from_logits);
  * 4-bit affine group-64 expert weights (Edge0, QuantSpec).
No page prints a dataset or a worked example; every value here is drawn from
a seeded generator.  bf16 values are produced by round-to-nearest-even from
fp32 draws (torch's ``.to(torch.bfloat16)``), so both sides read the same
bits.
"""
from __future__ import annotations

import copy
from dataclasses import dataclass, field, asdict
from typing import Optional

import numpy as np
import torch


@dataclass
class Workload:
    """Shape and options of one MoE layer forward (mirrors ``moe_config``)."""

    name: str
    T: int                      # tokens
    d: int                      # hidden
    F: int                      # expert intermediate
    E: int                      # routed experts
    k: int                      # top_k
    router: str = "softmax_topk"        # or "sigmoid_group"
    norm_topk_prob: bool = True
    routed_scaling: float = 1.0
    n_group: int = 1
    topk_group: int = 1
    capacity_factor: float = 0.0        # 0 => no capacity limit
    act: str = "swiglu"                 # or "relu"
    dtype: str = "bf16"                 # activation / weight dtype: f32 | bf16
    weight_format: str = "dense"        # dense | q4_affine_g64
    shared_F: int = 0                   # 0 => no shared expert
    aux_alpha: float = 0.01
    # input recipe
    x_std: float = 1.0
    w_std: float = 0.02
    router_std: float = 0.02
    logit_bias: str = "none"            # none | zipf1.1   (added to logits)
    selection_bias: float = 0.0         # U(-b, b) selection-only bias (sigmoid_group)
    tiny_numpy: bool = False            # use the numpy default_rng(0) recipe

    def with_(self, **kw) -> "Workload":
        w = copy.deepcopy(self)
        for key, val in kw.items():
            if not hasattr(w, key):
                raise AttributeError(key)
            setattr(w, key, val)
        return w

    def asdict(self) -> dict:
        return asdict(self)


WORKLOADS = {
    # T=64, d=16, E=4, top-2, softmax + renorm, ReLU d->32->d, cf=1.25, alpha 0.01,
    # N(0,1) tokens and N(0,1)*0.1 weights from numpy default_rng(0).
    "tiny_fp32": Workload("tiny_fp32", T=64, d=16, F=32, E=4, k=2, act="relu",
                          dtype="f32", capacity_factor=1.25, aux_alpha=0.01,
                          w_std=0.1, router_std=0.1, tiny_numpy=True),
    # Mixtral-style prefill, SwiGLU experts, no capacity limit.
    "mixtral_prefill": Workload("mixtral_prefill", T=4096, d=4096, F=14336, E=8, k=2,
                                act="swiglu"),
    # Switch-style top-1 with Zipf-skewed logits and cf = 1.0 (drops).
    "switch_top1": Workload("switch_top1", T=8192, d=2048, F=8192, E=64, k=1,
                            act="relu", capacity_factor=1.0, logit_bias="zipf1.1"),
    # DeepSeek-V3-style sigmoid group routing + one shared SwiGLU expert.
    "deepseek_v3": Workload("deepseek_v3", T=16384, d=7168, F=2048, E=256, k=8,
                            router="sigmoid_group", n_group=8, topk_group=4,
                            routed_scaling=2.5, norm_topk_prob=True,
                            selection_bias=0.05, shared_F=2048),
    # Decode-shaped 4-bit affine group-64 SwiGLU experts.
    "decode_q4": Workload("decode_q4", T=64, d=2048, F=768, E=128, k=8,
                          act="swiglu", weight_format="q4_affine_g64"),
}


def workload(name: str, **overrides) -> Workload:
    return WORKLOADS[name].with_(**overrides)


# ----------------------------------------------------------------------------
# draws

def _bf16(t: torch.Tensor) -> torch.Tensor:
    return t.to(torch.bfloat16)


def _randn(gen, shape, std, device, dtype):
    """N(0, std^2) drawn in fp32 then cast (RNE for bf16)."""
    t = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(dtype)


def zipf_logit_bias(E: int, s: float = 1.1) -> np.ndarray:
    """Fixed per-expert logit skew b_e = (e+1)^-s for e = 0..E-1 (max 1)."""
    return np.array([(e + 1.0) ** (-s) for e in range(E)], dtype=np.float32)


def make_inputs(w: Workload, seed: int = 0, device: str | torch.device = "cpu") -> dict:
    """Draw every input tensor of workload ``w``.

    Returns a dict of torch tensors on ``device``:
      x [T,d] (f32|bf16), w_router [E,d] f32, logit_bias [E] f32 or None,
      expert_bias [E] f32 or None (selection-only, sigmoid_group),
      dense weights: w_gate/w_in [E,F,d], w_up [E,F,d] (SwiGLU only), w_down/w_out [E,d,F];
      q4 weights: q_{gate,up,down} packed int32 codes, s_* / b_* bf16 per-64 scale / bias;
      shared expert: ws_gate [Fs,d], ws_up [Fs,d], ws_down [d,Fs].
    Keys for the first / last projection are always ``w1`` and ``w3`` (w2 = up).
    """
    device = torch.device(device)
    out: dict = {}
    if w.tiny_numpy:
        rng = np.random.default_rng(seed)
        x = rng.standard_normal((w.T, w.d))
        wr = rng.standard_normal((w.E, w.d)) * w.router_std
        w1 = rng.standard_normal((w.E, w.F, w.d)) * w.w_std
        w3 = rng.standard_normal((w.E, w.d, w.F)) * w.w_std
        w2 = rng.standard_normal((w.E, w.F, w.d)) * w.w_std if w.act == "swiglu" else None
        f = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device)
        out.update(x=f(x), w_router=f(wr), w1=f(w1), w3=f(w3), w2=f(w2) if w2 is not None else None)
    else:
        gen = torch.Generator(device=device)
        gen.manual_seed(seed)
        adt = torch.float32 if w.dtype == "f32" else torch.bfloat16
        out["x"] = _randn(gen, (w.T, w.d), w.x_std, device, adt)
        out["w_router"] = _randn(gen, (w.E, w.d), w.router_std, device, torch.float32)
        if w.weight_format == "dense":
            # one expert at a time keeps the fp32 temporary small
            def stack(n_rows, n_cols):
                t = torch.empty((w.E, n_rows, n_cols), device=device, dtype=adt)
                for e in range(w.E):
                    t[e] = _randn(gen, (n_rows, n_cols), w.w_std, device, adt)
                return t
            out["w1"] = stack(w.F, w.d)
            out["w2"] = stack(w.F, w.d) if w.act == "swiglu" else None
            out["w3"] = stack(w.d, w.F)
        else:
            out.update(make_q4_weights(w, gen, device))
        if w.shared_F:
            out["ws1"] = _randn(gen, (w.shared_F, w.d), w.w_std, device, adt)
            out["ws2"] = _randn(gen, (w.shared_F, w.d), w.w_std, device, adt)
            out["ws3"] = _randn(gen, (w.d, w.shared_F), w.w_std, device, adt)
        if w.selection_bias:
            b = torch.rand((w.E,), generator=gen, device=device, dtype=torch.float32)
            out["expert_bias"] = (b * 2.0 - 1.0) * w.selection_bias
    if w.logit_bias == "zipf1.1":
        out["logit_bias"] = torch.from_numpy(zipf_logit_bias(w.E, 1.1)).to(device)
    out.setdefault("expert_bias", None)
    out.setdefault("logit_bias", None)
    out.setdefault("w2", None)
    return out


def make_q4_weights(w: Workload, gen: torch.Generator, device) -> dict:
    """4-bit affine group-64 expert weights (Edge0 QuantSpec bits=4, group_size=64).

    Codes are uniform on 0..15, packed 8 per 32-bit word with element j of a
    row at bits 4*(j%8) of word j//8.  Per-group scale ~ N(0.02, 0.005) in
    bf16 and bias = bf16(-8 * scale), one pair per 64 consecutive elements of
    the reduction axis of each output row.
    Shapes: gate/up codes [E,F,d/8] int32, down codes [E,d,F/8] int32;
    scales/biases [E,N,K/64] bf16.
    """
    out = {}
    for key, (n, kdim) in (("1", (w.F, w.d)), ("2", (w.F, w.d)), ("3", (w.d, w.F))):
        codes = torch.randint(0, 16, (w.E, n, kdim), generator=gen, device=device, dtype=torch.int64)
        shifts = torch.arange(8, device=device, dtype=torch.int64) * 4
        packed = (codes.view(w.E, n, kdim // 8, 8) << shifts).sum(dim=-1)   # in [0, 2^32)
        packed = torch.where(packed >= 2**31, packed - 2**32, packed).to(torch.int32)
        scale = torch.randn((w.E, n, kdim // 64), generator=gen, device=device, dtype=torch.float32)
        scale = (scale * 0.005 + 0.02).to(torch.bfloat16)
        bias = (scale.float() * -8.0).to(torch.bfloat16)
        out["q" + key] = packed.contiguous()
        out["s" + key] = scale.contiguous()
        out["b" + key] = bias.contiguous()
    return out


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """The raw uint16 bit patterns of a bf16 tensor (host copy)."""
    assert t.dtype == torch.bfloat16
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def to_host(t: Optional[torch.Tensor]):
    """Host numpy view of an input: uint16 bits for bf16, else the array itself."""
    if t is None:
        return None
    if t.dtype == torch.bfloat16:
        return bf16_bits(t)
    return t.detach().cpu().contiguous().numpy()
