"""The single-token entry point that allocates nothing (library-owned scratch)
against the workspace entry point, on two calls in a row.

Collected last on purpose: a failure here leaves every other test run."""
import pytest
import torch

from mixed_precision_decode_b200 import bitsmoe as B
from mixed_precision_decode_b200 import synth
from mixed_precision_decode_b200.layer import PackedProjection, SpectralMoELayer

pytestmark = pytest.mark.gpu

TOL = 2e-3  # the parity tolerance of the other GPU tests


def _rel(a, b):
    return float(((a - b).abs().amax(-1) / b.abs().amax(-1).clamp_min(1e-30)).max())


def test_noalloc_matches_workspace_entry_point_twice():
    cfg = synth.CONFIGS["qwen_t1"]
    dev = torch.device("cuda")
    gen = synth.make_generator(4242, dev)
    projs = {}
    for name in ("gate", "up"):
        P = synth.make_projection(cfg, gen, dev)
        projs[name] = PackedProjection.from_factors(P["phi_t"], P["amps"], P["comps"], P["widths"], cfg.top_k)
        del P
    layer = SpectralMoELayer(projs["gate"], projs["up"])
    x = torch.randn((2, cfg.d_in), generator=gen, device=dev).to(torch.float16)
    ids, gw = synth.make_routing(cfg, gen, dev, 2)
    for t in range(2):  # two calls in a row, each on its own token and routing
        xt, it, gt = x[t:t + 1].contiguous(), ids[t:t + 1].contiguous(), gw[t:t + 1].contiguous()
        ref = layer.forward(xt, it, gt, want_experts=True)
        out = {k: torch.full_like(v, float("nan")) for k, v in ref.items()}
        ios = [B.proj_io(p.plan, p.blob, p.phi_t, out[f"Y_sum_{n}"], None, out[f"Y_experts_{n}"])
               for n, p in (("gate", projs["gate"]), ("up", projs["up"]))]
        st = torch.zeros(1, dtype=torch.int32, device=dev)
        B.layer_forward_t1_noalloc(ios[0], ios[1], xt, it, gt, st)
        assert B.read_status(st) == 0
        for k in ref:
            assert _rel(out[k], ref[k]) <= TOL, (t, k)
