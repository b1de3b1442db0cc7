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


def _layer(cfg, seed):
    dev = torch.device("cuda")
    gen = synth.make_generator(seed, dev)
    projs = {}
    for name in ("gate", "up"):
        P = synth.make_projection(cfg, gen, dev)
        projs[name] = PackedProjection.from_factors(P["phi_t"], P["amps"], P["comps"], P["widths"], cfg.top_k)
        del P
    x = torch.randn((1, cfg.d_in), generator=gen, device=dev).to(torch.float16)
    ids, gw = synth.make_routing(cfg, gen, dev, 1)
    return SpectralMoELayer(projs["gate"], projs["up"]), projs, x, ids, gw


def _noalloc_vs_workspace(layer, projs, x, ids, gw):
    ref = layer.forward(x, ids, gw, want_experts=True)
    out = {k: torch.full_like(v, float("nan")) for k, v in ref.items()}
    ios = [B.proj_io(p.plan, p.blob, p.phi_t, out[f"Y_sum_{n}"], None, out[f"Y_experts_{n}"])
           for n, p in (("gate", projs["gate"]), ("up", projs["up"]))]
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    B.layer_forward_t1_noalloc(ios[0], ios[1], x, ids, gw, st)
    assert B.read_status(st) == 0
    return max(_rel(out[k], ref[k]) for k in ref)


def test_noalloc_shapes_alternate_on_the_shared_scratch():
    """Calls of different shapes share the one scratch array: a Qwen-shaped layer
    (rank 2048), a smaller layer (rank 96, 40 rows, 6 experts), the Qwen layer
    again.  The smaller call's z rows stay in the array below the larger call's,
    and every result matches the workspace entry point."""
    big = _layer(synth.CONFIGS["qwen_t1"], 4343)
    small_cfg = synth.LayerConfig("noalloc_small", 128, 40, 6, 3, 96, 1,
                                  ((16, .1), (8, .1), (4, .2), (2, .4), (1, .1), (0, .1)), seed=4444)
    small = _layer(small_cfg, 4444)
    for lay in (big, small, big, small):
        assert _noalloc_vs_workspace(*lay) <= TOL
