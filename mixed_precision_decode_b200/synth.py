"""Seeded synthetic inputs for the spectral MoE gate/up layer.

This module holds input recipes only -- random draws, shapes and the
quantile rule that assigns widths -- and none of the method's arithmetic (no
scale, quantiser, packing or projection).  Both the CUDA path's tests/bench and
the oracle consume the tensors it returns (the oracle gets host copies), so no
value is ever generated twice by two different generators.

Workloads (shapes of the real models the BitsMoE pages evaluate, random
weights; no checkpoint or dataset is involved):

* ``tiny``        d_in 64, d_out 32, E 4, top-2, r 64, T 4, eight components at
                  each width 16/8/6/4/3/2/1/0.
* ``qwen_t1``     Qwen3-30B-A3B-shaped MoE layer (d_in 2048, d_out 768, E 128,
                  top-8, r 2048), one decode token, ~2.08 bits.
* ``qwen_t64``    same layer, 64 decode tokens, uniform random top-8, ~2.5 bits.
* ``qwen_stack``  48 independent ``qwen_t1``-style layers at T = 1, 8 or 32.
* ``mixtral_t16`` Mixtral-8x7B-shaped layer (d_in 4096, d_out 14336, E 8,
                  top-2, r 4096), 16 tokens, Zipf(1.2)-skewed routing, ~3.05 bits.

Recipe per projection (gate, then up): Phi = Q of a QR of an N(0,1) d_in x r
matrix (stored fp16, rows of ``phi_t`` are phi_k); a_{e,k} = k^-alpha *
LogNormal(0, sigma) with k 1-based; p_{e,k} = an N(0,1) d_out-vector divided by
its norm; widths assigned inside each expert by descending a (stable: lower k
first on ties) with counts n_b = round(F_b r) - round(F_{b-} r) from the
cumulative fractions F.  Then x ~ N(0,1) in fp16, then the routing draw.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace

import torch

WIDTH_SET = (0, 1, 2, 3, 4, 6, 8, 16)


@dataclass(frozen=True)
class LayerConfig:
    name: str
    d_in: int
    d_out: int
    n_experts: int
    top_k: int
    rank: int
    tokens: int
    # (width, fraction) in order of descending amplitude; fractions sum to 1
    width_fracs: tuple = field(default_factory=tuple)
    amp_power: float = 0.5
    amp_sigma: float = 0.5
    routing: str = "softmax_topk"  # softmax_topk | uniform | zipf
    zipf_s: float = 1.2
    seed: int = 0
    layers: int = 1


CONFIGS = {
    "tiny": LayerConfig("tiny", 64, 32, 4, 2, 64, 4,
                        tuple((b, 1 / 8) for b in (16, 8, 6, 4, 3, 2, 1, 0)),
                        amp_power=0.5, amp_sigma=0.3, seed=0),
    "qwen_t1": LayerConfig("qwen_t1", 2048, 768, 128, 8, 2048, 1,
                           ((8, .02), (4, .08), (3, .20), (2, .40), (1, .20), (0, .10)), seed=2),
    "qwen_t64": LayerConfig("qwen_t64", 2048, 768, 128, 8, 2048, 64,
                            ((16, .005), (8, .04), (4, .10), (3, .25), (2, .40), (1, .15), (0, .055)),
                            routing="uniform", seed=3),
    "qwen_stack": LayerConfig("qwen_stack", 2048, 768, 128, 8, 2048, 1,
                              ((8, .02), (4, .08), (3, .20), (2, .40), (1, .20), (0, .10)), seed=1000,
                              layers=48),
    "mixtral_t16": LayerConfig("mixtral_t16", 4096, 14336, 8, 2, 4096, 16,
                               ((8, .05), (4, .20), (3, .45), (2, .20), (1, .10)),
                               amp_power=0.7, amp_sigma=0.5, routing="zipf", zipf_s=1.2, seed=5),
}


def width_counts(cfg: LayerConfig) -> list[tuple[int, int]]:
    """(width, count) by cumulative rounding of the fractions (round half up)."""
    out, cum, prev = [], 0.0, 0
    for b, f in cfg.width_fracs:
        cum += f
        upto = int(math.floor(cum * cfg.rank + 0.5))
        upto = min(upto, cfg.rank)
        out.append((b, upto - prev))
        prev = upto
    if prev != cfg.rank:  # fractions that do not reach 1 leave the rest at width 0
        out.append((0, cfg.rank - prev))
    return out


def assign_widths(amps: torch.Tensor, counts: list[tuple[int, int]]) -> torch.Tensor:
    """widths [E][r] (uint8): inside each expert, by descending a, stable."""
    E, r = amps.shape
    order = torch.sort(amps.double(), dim=1, descending=True, stable=True).indices
    seq = torch.cat([torch.full((n,), b, dtype=torch.uint8) for b, n in counts]).to(amps.device)
    widths = torch.empty((E, r), dtype=torch.uint8, device=amps.device)
    widths.scatter_(1, order, seq.unsqueeze(0).expand(E, r).contiguous())
    return widths


def make_generator(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def make_projection(cfg: LayerConfig, gen: torch.Generator, device, experts=None) -> dict:
    """One projection's factors: phi_t [r][d_in] fp16, amps [E][r] f32,
    comps [E][r][d_out] f32 (unit rows), widths [E][r] u8."""
    d_in, d_out, E, r = cfg.d_in, cfg.d_out, cfg.n_experts, cfg.rank
    if r > d_in:
        raise ValueError(f"rank {r} > d_in {d_in}: an orthonormal basis of the input space has at most d_in columns")
    A = torch.randn((d_in, r), generator=gen, device=device, dtype=torch.float32)
    Q, _ = torch.linalg.qr(A)
    phi_t = Q.T.contiguous().to(torch.float16)
    k = torch.arange(1, r + 1, device=device, dtype=torch.float32)
    ln = torch.exp(cfg.amp_sigma * torch.randn((E, r), generator=gen, device=device, dtype=torch.float32))
    amps = (k.pow(-cfg.amp_power).unsqueeze(0) * ln).contiguous()
    comps = torch.randn((E, r, d_out), generator=gen, device=device, dtype=torch.float32)
    comps /= torch.linalg.vector_norm(comps, dim=2, keepdim=True)
    widths = assign_widths(amps, width_counts(cfg))
    return {"phi_t": phi_t, "amps": amps, "comps": comps, "widths": widths}


def make_down(cfg: LayerConfig, gen: torch.Generator, device) -> torch.Tensor:
    """Dense down-projection weights of every expert, w_down [E][d_in][d_out] fp16:
    N(0, 1) / sqrt(d_out) (fan-in scaling), one expert at a time."""
    E, d_model, d_ff = cfg.n_experts, cfg.d_in, cfg.d_out
    w = torch.empty((E, d_model, d_ff), dtype=torch.float16, device=device)
    for e in range(E):
        w[e] = (torch.randn((d_model, d_ff), generator=gen, device=device, dtype=torch.float32)
                * d_ff ** -0.5).to(torch.float16)
    return w


def make_routing(cfg: LayerConfig, gen: torch.Generator, device, tokens: int) -> tuple[torch.Tensor, torch.Tensor]:
    """(ids [T][top_k] int32, gate weights [T][top_k] f32)."""
    E, k, T = cfg.n_experts, cfg.top_k, tokens
    if cfg.routing == "softmax_topk":
        logits = torch.randn((T, E), generator=gen, device=device, dtype=torch.float32)
        probs = torch.softmax(logits, dim=1)
        vals, ids = torch.topk(probs, k, dim=1)
        w = vals / vals.sum(dim=1, keepdim=True)
    elif cfg.routing == "uniform":
        ids = torch.rand((T, E), generator=gen, device=device).argsort(dim=1)[:, :k]
        w = torch.softmax(torch.randn((T, k), generator=gen, device=device, dtype=torch.float32), dim=1)
    elif cfg.routing == "zipf":
        pe = torch.arange(1, E + 1, device=device, dtype=torch.float64).pow(-cfg.zipf_s)
        pe = (pe / pe.sum()).float()
        ids = torch.multinomial(pe.unsqueeze(0).expand(T, E).contiguous(), k, replacement=False, generator=gen)
        w = torch.softmax(torch.randn((T, k), generator=gen, device=device, dtype=torch.float32), dim=1)
    else:
        raise ValueError(cfg.routing)
    return ids.to(torch.int32).contiguous(), w.float().contiguous()


def make_layer(cfg: LayerConfig, seed: int | None = None, device="cpu", tokens: int | None = None) -> dict:
    """A full synthetic layer: gate and up projections, tokens and routing."""
    seed = cfg.seed if seed is None else seed
    T = cfg.tokens if tokens is None else tokens
    gen = make_generator(seed, device)
    gate = make_projection(cfg, gen, device)
    up = make_projection(cfg, gen, device)
    x = torch.randn((T, cfg.d_in), generator=gen, device=device, dtype=torch.float32).to(torch.float16)
    ids, w = make_routing(cfg, gen, device, T)
    return {"cfg": cfg, "seed": seed, "gate": gate, "up": up, "x": x, "ids": ids, "gate_w": w}


def scaled(cfg: LayerConfig, **kw) -> LayerConfig:
    """A copy of ``cfg`` with some fields replaced (smaller parity cases)."""
    return replace(cfg, **kw)
