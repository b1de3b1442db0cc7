"""Parity cases shared by the GPU tests: seeded synthetic layers packed by the
CUDA path, plus host copies of exactly the tensors the oracle needs.

Full-size layers (Qwen3-30B-A3B- and Mixtral-shaped) are generated on the GPU;
the oracle gets host copies of the experts a test samples and packs those
alone (an expert's section of the blob depends only on that expert)."""
from __future__ import annotations

import functools

import numpy as np
import torch

from mixed_precision_decode_b200 import synth
from mixed_precision_decode_b200.layer import PackedProjection, SpectralMoELayer

TOL = 2e-3  # max relative error per output vector (fp32 accumulation vs fp64 oracle)

# Small cases the oracle finishes in seconds, spanning several row blocks,
# member chunks, a ragged row count and member padding.
SMALL = {
    "tiny": synth.CONFIGS["tiny"],
    "ragged": synth.LayerConfig("ragged", 96, 37, 6, 3, 77, 5,
                                ((16, .1), (8, .1), (6, .1), (4, .15), (3, .15), (2, .2), (1, .1), (0, .1)),
                                amp_power=0.5, amp_sigma=0.5, seed=7),
    "ragged_big": synth.LayerConfig("ragged_big", 3072, 600, 4, 2, 3000, 9,
                                    ((16, .01), (8, .04), (2, .6), (1, .3), (0, .05)),
                                    amp_power=0.5, amp_sigma=0.5, seed=8),
    "one_expert": synth.LayerConfig("one_expert", 64, 96, 1, 1, 50, 3,
                                    ((4, .5), (1, .5)), amp_power=0.5, amp_sigma=0.3, seed=9),
}
FULL = {k: synth.CONFIGS[k] for k in ("qwen_t1", "qwen_t64", "mixtral_t16")}


def rel_err(y: np.ndarray, ref: np.ndarray) -> float:
    """max over output vectors of max_i |y - ref| / max_i |ref| (last axis = rows)."""
    y = np.asarray(y, np.float64)
    ref = np.asarray(ref, np.float64)
    num = np.abs(y - ref).max(axis=-1)
    den = np.abs(ref).max(axis=-1)
    den = np.where(den > 0, den, 1.0)
    return float((num / den).max()) if num.size else 0.0


class Case:
    """One layer on the GPU + what the oracle needs, per projection."""

    def __init__(self, cfg: synth.LayerConfig):
        self.cfg = cfg
        self._oracle = {}
        dev = torch.device("cuda")
        gen = synth.make_generator(cfg.seed, dev)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        self.proj = {}
        self.host = {}
        for name in ("gate", "up"):
            P = synth.make_projection(cfg, gen, dev)
            pk = PackedProjection.from_factors(P["phi_t"], P["amps"], P["comps"], P["widths"], cfg.top_k,
                                               status=self.status)
            self.proj[name] = pk
            self.host[name] = {
                "phi_t": P["phi_t"].cpu().numpy().view(np.uint16),
                "widths": P["widths"].cpu().numpy(),
                "amps": P["amps"].cpu().numpy(),
                "comps_dev": P["comps"],  # the oracle copies out the experts it samples
            }
        self.x = torch.randn((cfg.tokens, cfg.d_in), generator=gen, device=dev).to(torch.float16)
        self.ids, self.gate_w = synth.make_routing(cfg, gen, dev, cfg.tokens)
        self.layer = SpectralMoELayer(self.proj["gate"], self.proj["up"])
        torch.cuda.synchronize()

    def comps_host(self, name: str, experts) -> np.ndarray:
        c = self.host[name]["comps_dev"]
        return c[torch.as_tensor(list(experts), device=c.device)].cpu().numpy()

    def oracle_blob(self, orc, name: str, experts):
        """Oracle blob of the given experts alone (in the given order), cached."""
        ex = tuple(int(e) for e in experts)
        key = (name, ex)
        if key not in self._oracle:
            comps = self.comps_host(name, ex)
            w = self.host[name]["widths"][list(ex)]
            a = self.host[name]["amps"][list(ex)]
            scales, st = orc.compute_scales(comps, w)
            blob, st2 = orc.pack(comps, w, scales, a)
            self._oracle[key] = (blob, scales, st | st2)
        return self._oracle[key]

    def gpu_blob(self, name: str) -> np.ndarray:
        return self.proj[name].blob.cpu().numpy()


def expert_section(blob: np.ndarray, e: int) -> np.ndarray:
    d = blob[64 + 64 * e: 128 + 64 * e]
    base = int(d[0:8].view(np.uint64)[0])
    n = int(d[8:16].view(np.uint64)[0])
    return blob[base:base + n]


@functools.lru_cache(maxsize=2)
def get_case(name: str) -> Case:
    if name in SMALL:
        return Case(SMALL[name])
    return Case(FULL[name])


def x_bits(case: Case) -> np.ndarray:
    return case.x.cpu().numpy().view(np.uint16)


def oracle_tokens(case: Case, orc, proj: str, toks, Z, ids=None, gate_w=None):
    """Oracle Y_e / Y_sum for the given tokens, on a blob of just their experts."""
    ids = (case.ids if ids is None else ids).cpu().numpy()[toks]
    g = (case.gate_w if gate_w is None else gate_w).cpu().numpy()[toks]
    ex = sorted(set(int(v) for v in ids.ravel()))
    remap = {e: j for j, e in enumerate(ex)}
    blob, _, _ = case.oracle_blob(orc, proj, ex)
    rid = np.vectorize(remap.get)(ids).astype(np.int32)
    Ye, Ys, st = orc.expert_forward(blob, Z, rid, g)
    assert st == 0
    return Ye, Ys
