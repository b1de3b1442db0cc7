"""Degenerate experts and routings against the oracle, on the single-token
fused kernel (T = 1) and the multi-token path (T > 1): an expert that stores no
component (every width 0), an expert of fp16 components only, and a token
whose top-k names the same expert twice."""
import numpy as np
import pytest
import torch

from cases import TOL, rel_err
from mixed_precision_decode_b200 import bitsmoe as B
from mixed_precision_decode_b200.layer import PackedProjection, SpectralMoELayer

pytestmark = pytest.mark.gpu

D_IN, D_OUT, E, K, R = 64, 40, 4, 2, 64


def _widths(rng):
    w = np.zeros((E, R), np.uint8)  # expert 0: every component dropped
    w[1] = 16                        # expert 1: fp16 components only
    for e in (2, 3):                 # experts 2, 3: every width
        w[e] = rng.choice(np.array([0, 1, 2, 3, 4, 6, 8, 16], np.uint8), size=R)
    return w


def _projection(rng, gen, w):
    a = torch.linalg.qr(torch.randn((D_IN, R), generator=gen, device="cuda"))[0]
    phi_t = a.T.contiguous().to(torch.float16)
    comps = torch.randn((E, R, D_OUT), generator=gen, device="cuda")
    comps = comps / comps.norm(dim=-1, keepdim=True)
    amps = torch.rand((E, R), generator=gen, device="cuda") + 0.1
    pk = PackedProjection.from_factors(phi_t, amps, comps, torch.as_tensor(w), K)
    host = {"phi_t": phi_t.cpu().numpy().view(np.uint16), "comps": comps.cpu().numpy(), "amps": amps.cpu().numpy()}
    return pk, host


@pytest.fixture(scope="module")
def layer():
    rng = np.random.default_rng(11)
    gen = torch.Generator(device="cuda").manual_seed(11)
    w = _widths(rng)
    projs, hosts = {}, {}
    for name in ("gate", "up"):
        projs[name], hosts[name] = _projection(rng, gen, w)
    return SpectralMoELayer(projs["gate"], projs["up"]), hosts, w


IDS = np.array([[0, 1], [2, 2], [3, 0], [1, 3], [2, 1]], np.int32)
GW = np.array([[0.7, 0.3], [0.6, 0.4], [0.5, 0.5], [0.2, 0.8], [0.9, 0.1]], np.float32)


@pytest.mark.parametrize("rows", [[0], [1], [0, 1, 2, 3, 4]], ids=["t1_dropped_and_fp16", "t1_same_expert_twice", "t5"])
def test_degenerate_experts_and_routings(layer, orc, rows):
    """Row 0: the all-dropped expert and the fp16-only one; row 1: expert 2 twice; the rest mixed."""
    lay, hosts, w = layer
    T = len(rows)
    gen = torch.Generator(device="cuda").manual_seed(100 + T)
    x = torch.randn((T, D_IN), generator=gen, device="cuda").to(torch.float16)
    ids, gw = IDS[rows], GW[rows]
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = lay.forward(x, torch.as_tensor(ids, device="cuda"), torch.as_tensor(gw, device="cuda"), want_experts=True,
                      status=st)
    assert B.read_status(st) == 0
    xb = x.cpu().numpy().view(np.uint16)
    for name in ("gate", "up"):
        h = hosts[name]
        scales, s0 = orc.compute_scales(h["comps"], w)
        blob, s1 = orc.pack(h["comps"], w, scales, h["amps"])
        assert s0 == 0 and s1 == 0
        Z = orc.shared_proj(h["phi_t"], xb)
        Ye_ref, Ys_ref, s2 = orc.expert_forward(blob, Z, ids, gw)
        assert s2 == 0
        Ye = out[f"Y_experts_{name}"].cpu().numpy()
        assert rel_err(Ye, Ye_ref) <= TOL
        assert rel_err(out[f"Y_sum_{name}"].cpu().numpy(), Ys_ref) <= TOL
        for t in range(T):  # the expert that stores nothing gives exactly zero
            for j in range(K):
                if ids[t, j] == 0:
                    assert np.all(Ye[t, j] == 0.0)
        for t in range(T):  # the same expert twice in one token: the same row twice, up to the order
            if ids[t, 0] == ids[t, 1]:  # of the fp32 additions (the fused path splits the two slots differently)
                assert rel_err(Ye[t, 0], Ye[t, 1]) <= 1e-5
