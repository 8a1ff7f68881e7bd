"""Seeded synthetic inputs for the sparse MoE feed-forward layer.

This module draws random numbers and rounds them to the storage dtypes; it
holds none of the layer's arithmetic (no routing, no FFN, no combine). Both the
CUDA path and the CPU oracle are fed from here, so they see bit-identical
inputs.

Recipe (one ``torch.Generator`` seeded with ``seed``, draws in this order):

1. per-expert logit bias ``b[E]`` (fp32): zero, N(0, 0.5) (Mixtral-shaped
   prefill) or ``-s*ln(e+1)`` (Zipf(s) popularity, skewed prefill);
2. router logits ``z[T,E]`` fp32 = N(0,1) + b, every row redrawn until the gap
   between its k-th and (k+1)-th largest value is at least ``margin`` (1e-3),
   so the top-k set is not decided by rounding;
3. hidden states ``x[T,H]`` = N(0,1) rounded to bf16;
4. ``per_expert_scale[E]`` fp32: ones or U[0.5, 1.5];
5. ``w13[E,2I,H]`` = N(0, 0.02) rounded to bf16, expert by expert (rows
   ``[0,I)`` are the gate projection w1, rows ``[I,2I)`` the up projection
   w3);
6. ``w2[E,H,I]`` = N(0, 0.02) rounded to bf16;
7. shared experts (if any) ``w13_sh[S,2Is,H]``, ``w2_sh[S,H,Is]`` likewise.

Weight layout follows the FusedMoE packing described on the vLLM API page
(vllm.model_executor.models.gemma4, ``load_weights``: gate_proj -> w1 and
up_proj -> w3 shards of ``w13_weight``, gate/up ``[I, H]``, down ``[H, I]``)
and the gated-FFN section of the "MOE Inference" blog (gaohongy.github.io,
"门控(Gated) FFN": ``[y1, y3] = x . [w1, w3]``).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch

ACT_SILU = 0
ACT_GELU_TANH = 1

# The workloads.  Shapes and distributions are those of the Gemma-4 26B-A4B
# MoE block (H=2816, E=128, k=8, I=704, tanh-GELU) and of Mixtral 8x7B
# (E=8, k=2) named on the pages, plus a tiny case and a skewed case with
# shared experts (llama-cpp-visual-guide lesson 35, "shared expert").
CONFIGS = {
    "tiny": dict(T=64, H=256, E=8, k=2, I=512, act=ACT_SILU,
                 bias="zero", scale="ones"),
    "mixtral_prefill": dict(T=4096, H=4096, E=8, k=2, I=14336, act=ACT_SILU,
                            bias="normal0.5", scale="ones"),
    "many_small_prefill": dict(T=8192, H=2816, E=128, k=8, I=704,
                               act=ACT_GELU_TANH, bias="zero", scale="uniform"),
    "skewed_shared_prefill": dict(T=16384, H=2048, E=64, k=6, I=1408,
                                  act=ACT_SILU, n_shared=2, I_shared=1408,
                                  bias="zipf1.1", scale="ones"),
}
for _t in (1, 4, 16, 64, 256):
    CONFIGS[f"decode_t{_t}"] = dict(T=_t, H=2816, E=128, k=8, I=704,
                                    act=ACT_GELU_TANH, bias="zero",
                                    scale="uniform")


@dataclasses.dataclass
class Shape:
    T: int
    H: int
    E: int
    k: int
    I: int
    act: int = ACT_SILU
    n_shared: int = 0
    I_shared: int = 0
    pad: int = 128

    @property
    def rows(self) -> int:
        """Routed (token, expert) rows, T*k."""
        return self.T * self.k

    def flops(self) -> float:
        """Algorithmic FLOPs: 6*H*I per real routed row plus 6*H*Is per
        shared row; tile padding is never counted."""
        f = 6.0 * self.H * self.I * self.T * self.k
        f += 6.0 * self.H * self.I_shared * self.T * self.n_shared
        return f


@dataclasses.dataclass
class MoEInputs:
    shape: Shape
    x: torch.Tensor            # [T,H] bf16
    logits: torch.Tensor       # [T,E] fp32
    scale: torch.Tensor        # [E] fp32
    w13: torch.Tensor          # [E,2I,H] bf16
    w2: torch.Tensor           # [E,H,I] bf16
    w13_sh: Optional[torch.Tensor] = None  # [S,2Is,H] bf16
    w2_sh: Optional[torch.Tensor] = None   # [S,H,Is] bf16
    bias: Optional[torch.Tensor] = None    # [E] fp32 (generator detail)


def shape_of(name: str, **overrides) -> Shape:
    cfg = dict(CONFIGS[name])
    cfg.update(overrides)
    return Shape(T=cfg["T"], H=cfg["H"], E=cfg["E"], k=cfg["k"], I=cfg["I"],
                 act=cfg["act"], n_shared=cfg.get("n_shared", 0),
                 I_shared=cfg.get("I_shared", 0))


def _bias(kind: str, E: int, gen: torch.Generator, device) -> torch.Tensor:
    if kind == "zero":
        return torch.zeros(E, dtype=torch.float32, device=device)
    if kind == "normal0.5":
        return 0.5 * torch.randn(E, generator=gen, device=device,
                                 dtype=torch.float32)
    if kind.startswith("zipf"):
        s = float(kind[4:])
        e = torch.arange(E, dtype=torch.float64, device=device)
        return (-s * torch.log(e + 1.0)).to(torch.float32)
    raise ValueError(f"unknown bias kind {kind!r}")


def router_logits(T: int, E: int, k: int, gen: torch.Generator, device,
                  bias: Optional[torch.Tensor] = None,
                  margin: float = 1e-3, max_rounds: int = 1000) -> torch.Tensor:
    """N(0,1) (+bias) fp32 logits, each row redrawn until the k-th and
    (k+1)-th largest values differ by at least ``margin``."""
    if bias is None:
        bias = torch.zeros(E, dtype=torch.float32, device=device)
    z = torch.randn(T, E, generator=gen, device=device, dtype=torch.float32)
    z = z + bias
    if k >= E or T == 0:
        return z.contiguous()
    for _ in range(max_rounds):
        top = torch.topk(z, k + 1, dim=-1).values
        bad = (top[:, k - 1] - top[:, k]) < margin
        nbad = int(bad.sum())
        if nbad == 0:
            return z.contiguous()
        fresh = torch.randn(nbad, E, generator=gen, device=device,
                            dtype=torch.float32) + bias
        z[bad] = fresh
    raise RuntimeError("could not meet the top-k margin")


def router_inputs(T: int, H: int, E: int, gen: torch.Generator, device):
    """Inputs of the router ahead of the routing: the residual rows [T,H]
    (N(0, 4) in bf16 -- the router normalises them away), the GateLinear
    weight [E,H] (N(0,1) in bf16, so that the logits come out near unit
    scale) and the per-dimension scale [H] (U[0.5, 1.5] in bf16)."""
    x = (2.0 * torch.randn(T, H, generator=gen, device=device)).to(torch.bfloat16)
    w = torch.randn(E, H, generator=gen, device=device).to(torch.bfloat16)
    s = (0.5 + torch.rand(H, generator=gen, device=device)).to(torch.bfloat16)
    return x.contiguous(), w.contiguous(), s.contiguous()


def _normal_bf16(shape, std: float, gen: torch.Generator, device) -> torch.Tensor:
    out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    if out.dim() == 3:
        # expert by expert keeps the fp32 temporary small
        for e in range(out.shape[0]):
            t = torch.randn(out.shape[1:], generator=gen, device=device,
                            dtype=torch.float32)
            out[e].copy_((t * std).to(torch.bfloat16))
    else:
        t = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
        out.copy_((t * std).to(torch.bfloat16))
    return out


def make_inputs(name_or_shape, seed: int = 0, device="cpu",
                bias: Optional[str] = None, scale: Optional[str] = None,
                **overrides) -> MoEInputs:
    """Build one workload.  ``name_or_shape`` is a key of ``CONFIGS`` or a
    ``Shape`` (then ``bias``/``scale`` pick the distributions)."""
    if isinstance(name_or_shape, Shape):
        shp = name_or_shape
        bias_kind = bias or "zero"
        scale_kind = scale or "ones"
    else:
        cfg = CONFIGS[name_or_shape]
        shp = shape_of(name_or_shape, **overrides)
        bias_kind = bias or cfg.get("bias", "zero")
        scale_kind = scale or cfg.get("scale", "ones")
    device = torch.device(device)
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    b = _bias(bias_kind, shp.E, gen, device)
    z = router_logits(shp.T, shp.E, shp.k, gen, device, bias=b)
    x = _normal_bf16((shp.T, shp.H), 1.0, gen, device)
    if scale_kind == "ones":
        sc = torch.ones(shp.E, dtype=torch.float32, device=device)
    elif scale_kind == "uniform":
        sc = 0.5 + torch.rand(shp.E, generator=gen, device=device,
                              dtype=torch.float32)
    else:
        raise ValueError(f"unknown scale kind {scale_kind!r}")
    w13 = _normal_bf16((shp.E, 2 * shp.I, shp.H), 0.02, gen, device)
    w2 = _normal_bf16((shp.E, shp.H, shp.I), 0.02, gen, device)
    w13_sh = w2_sh = None
    if shp.n_shared:
        w13_sh = _normal_bf16((shp.n_shared, 2 * shp.I_shared, shp.H), 0.02,
                              gen, device)
        w2_sh = _normal_bf16((shp.n_shared, shp.H, shp.I_shared), 0.02,
                             gen, device)
    return MoEInputs(shape=shp, x=x, logits=z, scale=sc, w13=w13, w2=w2,
                     w13_sh=w13_sh, w2_sh=w2_sh, bias=b)


def zipf_weights(E: int, s: float) -> list:
    """Normalised Zipf(s) popularity over E ranks (for reports only)."""
    w = [(e + 1.0) ** (-s) for e in range(E)]
    tot = math.fsum(w)
    return [v / tot for v in w]


@dataclasses.dataclass
class Gemma4BlockInputs:
    """Inputs of the Gemma 4 MoE block beyond the experts (``MoEInputs``):
    the residual rows, the five gamma vectors, the dense MLP and the router."""
    x: torch.Tensor            # [T,H] bf16 residual (the MoE experts' weights come
                               # from MoEInputs; its x and logits are not used)
    norms: tuple               # 5 x [H] bf16: pre_ff, post_ff_1, pre_ff_2, post_ff_2, post_ff
    mlp_w13: torch.Tensor      # [2*I_dense, H] bf16, gate rows first
    mlp_w2: torch.Tensor       # [H, I_dense] bf16
    router_w: torch.Tensor     # [E,H] bf16
    router_scale: torch.Tensor  # [H] bf16


def gemma4_block_inputs(T: int, H: int, E: int, I_dense: int, seed: int = 0,
                        device="cpu") -> Gemma4BlockInputs:
    """Recipe (one generator seeded with ``seed``, in this order): residual
    rows N(0,1) -> bf16; the five gammas 1 + N(0, 0.1) -> bf16; the dense
    MLP's w13 [2*I_dense, H] and w2 [H, I_dense] N(0, 0.02) -> bf16; the
    router's GateLinear weight N(0,1) -> bf16 (logits near unit scale, as in
    ``router_inputs``); the router scale U[0.5, 1.5] -> bf16."""
    device = torch.device(device)
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    x = _normal_bf16((T, H), 1.0, gen, device)
    norms = tuple((1.0 + 0.1 * torch.randn(H, generator=gen, device=device))
                  .to(torch.bfloat16) for _ in range(5))
    mlp_w13 = _normal_bf16((2 * I_dense, H), 0.02, gen, device)
    mlp_w2 = _normal_bf16((H, I_dense), 0.02, gen, device)
    rw = torch.randn(E, H, generator=gen, device=device).to(torch.bfloat16)
    rs = (0.5 + torch.rand(H, generator=gen, device=device)).to(torch.bfloat16)
    return Gemma4BlockInputs(x=x, norms=norms, mlp_w13=mlp_w13, mlp_w2=mlp_w2,
                             router_w=rw, router_scale=rs)


@dataclasses.dataclass
class FP8Experts:
    """Expert weights as e4m3 codes (uint8) with one fp32 scale per output
    row: the per-expert FP8 checkpoints' weight / weight_scale pairs, packed
    as w13 (gate rows first) and w2."""
    w13_q: torch.Tensor                     # [E,2I,H] uint8
    w13_s: torch.Tensor                     # [E,2I] fp32
    w2_q: torch.Tensor                      # [E,H,I] uint8
    w2_s: torch.Tensor                      # [E,H] fp32
    sh13_q: Optional[torch.Tensor] = None   # [S,2I,H] uint8
    sh13_s: Optional[torch.Tensor] = None   # [S,2I] fp32
    sh2_q: Optional[torch.Tensor] = None    # [S,H,I] uint8
    sh2_s: Optional[torch.Tensor] = None    # [S,H] fp32


def _e4m3_codes(shape, gen: torch.Generator, device) -> torch.Tensor:
    """N(0, 64^2) draws clamped to the e4m3 range and rounded to e4m3 (torch's
    float8_e4m3fn cast), as uint8 codes; 3-d tensors expert by expert."""
    out = torch.empty(shape, dtype=torch.uint8, device=device)
    parts = [out[e] for e in range(shape[0])] if len(shape) == 3 else [out]
    for o in parts:
        t = torch.randn(o.shape, generator=gen, device=device, dtype=torch.float32)
        o.copy_((64.0 * t).clamp_(-448.0, 448.0).to(torch.float8_e4m3fn)
                .view(torch.uint8))
    return out


def _row_scales(shape, gen: torch.Generator, device) -> torch.Tensor:
    return ((0.5 + torch.rand(shape, generator=gen, device=device,
                              dtype=torch.float32)) * (0.02 / 64.0)).contiguous()


def fp8_experts(shp: Shape, seed: int = 0, device="cpu") -> FP8Experts:
    """Recipe (one generator seeded with ``seed``, draws in this order): w13
    codes, w13 row scales, w2 codes, w2 row scales, then the shared experts'
    in the same order.  Codes are e4m3 roundings of N(0, 64^2) draws, scales
    (0.5 + U[0,1]) * 0.02 / 64, so the weights they stand for spread like the
    bf16 recipe's N(0, 0.02^2)."""
    device = torch.device(device)
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    E, H, I, S = shp.E, shp.H, shp.I, shp.n_shared
    w13_q = _e4m3_codes((E, 2 * I, H), gen, device)
    w13_s = _row_scales((E, 2 * I), gen, device)
    w2_q = _e4m3_codes((E, H, I), gen, device)
    w2_s = _row_scales((E, H), gen, device)
    sh = [None] * 4
    if S:
        sh = [_e4m3_codes((S, 2 * I, H), gen, device), _row_scales((S, 2 * I), gen, device),
              _e4m3_codes((S, H, I), gen, device), _row_scales((S, H), gen, device)]
    return FP8Experts(w13_q, w13_s, w2_q, w2_s, *sh)
