"""Properties of the CUDA path that hold at any size (closed forms and
invariants), plus its data-error reporting.  None of these inputs faults."""
import numpy as np
import pytest
import torch

from cases import TOL, get_case, rel_err
from mixed_precision_decode_b200 import bitsmoe as B
from mixed_precision_decode_b200 import synth
from mixed_precision_decode_b200.layer import PackedProjection, SpectralMoELayer

pytestmark = pytest.mark.gpu


def test_shared_proj_identity_and_one_hot():
    """Phi = I gives Z = x exactly; a one-hot x gives a column of Phi^T exactly."""
    d = 256
    eye = torch.eye(d, dtype=torch.float16, device="cuda")
    x = torch.randn((5, d), device="cuda").to(torch.float16)
    Z = torch.empty((5, d), dtype=torch.float32, device="cuda")
    B.shared_proj(eye, x, Z, 5, d, d)
    assert torch.equal(Z, x.float())
    phi_t = torch.randn((300, d), device="cuda").to(torch.float16)
    oh = torch.zeros((1, d), dtype=torch.float16, device="cuda")
    oh[0, 77] = 1
    Z = torch.empty((1, 300), dtype=torch.float32, device="cuda")
    B.shared_proj(phi_t, oh, Z, 1, d, 300)
    assert torch.equal(Z[0], phi_t[:, 77].float())


@pytest.mark.parametrize("name", ["ragged", "qwen_t64"])
def test_routing_invariants(name):
    """Slot permutation permutes Y_e exactly and keeps Y_sum; doubling g doubles
    Y_sum exactly; a token alone matches the same token inside the batch."""
    case = get_case(name)
    lay = case.layer
    out = lay.forward(case.x, case.ids, case.gate_w, want_experts=True)
    perm = torch.randperm(case.cfg.top_k, generator=torch.Generator().manual_seed(1)).cuda()
    out_p = lay.forward(case.x, case.ids[:, perm].contiguous(), case.gate_w[:, perm].contiguous(),
                        want_experts=True)
    out_2 = lay.forward(case.x, case.ids, (2 * case.gate_w).contiguous(), want_experts=True)
    for proj in ("gate", "up"):
        assert torch.equal(out_p[f"Y_experts_{proj}"], out[f"Y_experts_{proj}"][:, perm])
        assert rel_err(out_p[f"Y_sum_{proj}"].cpu().numpy(), out[f"Y_sum_{proj}"].cpu().numpy()) <= 1e-5
        assert torch.equal(out_2[f"Y_sum_{proj}"], 2 * out[f"Y_sum_{proj}"])
    t = case.cfg.tokens // 2
    one = lay.forward(case.x[t:t + 1].contiguous(), case.ids[t:t + 1].contiguous(),
                      case.gate_w[t:t + 1].contiguous(), want_experts=True)
    for proj in ("gate", "up"):
        assert rel_err(one[f"Y_sum_{proj}"].cpu().numpy(), out[f"Y_sum_{proj}"][t:t + 1].cpu().numpy()) <= 1e-5
        assert rel_err(one[f"Y_experts_{proj}"].cpu().numpy(),
                       out[f"Y_experts_{proj}"][t:t + 1].cpu().numpy()) <= 1e-5


def test_bad_expert_id_sets_status_and_zeroes_row():
    case = get_case("ragged")
    ids = case.ids.clone()
    ids[1, 0] = case.cfg.n_experts + 3
    ids[2, 1] = -1
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = case.layer.forward(case.x, ids, case.gate_w, want_experts=True, status=st)
    assert B.read_status(st) & B.ST_BADEXPERT
    ref = case.layer.forward(case.x, case.ids, case.gate_w, want_experts=True)
    for proj in ("gate", "up"):
        Ye = out[f"Y_experts_{proj}"]
        assert torch.all(Ye[1, 0] == 0) and torch.all(Ye[2, 1] == 0)
        g = case.gate_w
        expect = sum(g[1, j] * ref[f"Y_experts_{proj}"][1, j] for j in range(1, case.cfg.top_k))
        assert rel_err(out[f"Y_sum_{proj}"][1].cpu().numpy(), expect.cpu().numpy()) <= 1e-5


def test_zero_tokens_is_a_noop():
    case = get_case("tiny")
    out = case.layer.forward(case.x[:0], case.ids[:0], case.gate_w[:0])
    assert out["Y_sum_gate"].shape == (0, case.cfg.d_out)


def test_nonfinite_component_and_bad_scale_are_reported():
    cfg = synth.scaled(synth.CONFIGS["tiny"], seed=11)
    P = synth.make_projection(cfg, synth.make_generator(11, "cuda"), "cuda")
    comps = P["comps"].clone()
    w = P["widths"]
    e, k = 1, int(torch.nonzero(w[1] == 2)[0])
    comps[e, k, 3] = float("nan")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    pk = PackedProjection.from_factors(P["phi_t"], P["amps"], comps, w, cfg.top_k, status=st)
    assert B.read_status(st) & B.ST_NONFINITE
    # a negative caller scale: its q are 0 and the bad-scale bit is set
    scales = torch.full(w.shape, 0x3800, dtype=torch.int16, device="cuda")
    scales[0, int(torch.nonzero(w[0] == 3)[0])] = np.int16(np.uint16(0xB800).view(np.int16))
    st2 = torch.zeros(1, dtype=torch.int32, device="cuda")
    PackedProjection.from_factors(P["phi_t"], P["amps"], P["comps"], w, cfg.top_k, scales=scales, status=st2)
    assert B.read_status(st2) & B.ST_BADSCALE


def test_plan_mismatch_is_reported_not_faulted():
    cfg = synth.CONFIGS["tiny"]
    P = synth.make_projection(cfg, synth.make_generator(3, "cuda"), "cuda")
    plan = B.pack_plan(cfg.d_in, cfg.d_out, cfg.n_experts, cfg.rank, cfg.top_k, P["widths"].cpu())
    other = P["widths"].clone()
    other[0, int(torch.nonzero(other[0] == 2)[0])] = 3  # the device widths now disagree with the plan
    blob = torch.empty(plan.blob_bytes, dtype=torch.uint8, device="cuda")
    scales = torch.zeros(P["widths"].shape, dtype=torch.int16, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    B.pack(plan, P["comps"], other.contiguous(), scales, P["amps"], blob, st)
    assert B.read_status(st) & B.ST_PLANMISMATCH


def test_blob_save_and_reload(tmp_path):
    """A blob saved to disk and reloaded (plan rebuilt from its header) gives
    the same outputs."""
    case = get_case("tiny")
    pk = case.proj["gate"]
    path = tmp_path / "gate.blob"
    pk.blob.cpu().numpy().tofile(path)
    data = np.fromfile(path, np.uint8)
    plan = B.plan_from_header(data[:pk.plan.header_bytes], case.cfg.d_in, case.cfg.top_k)
    pk2 = PackedProjection(plan, torch.as_tensor(data, device="cuda"), pk.phi_t)
    lay2 = SpectralMoELayer(pk2, case.proj["up"])
    a = case.layer.forward(case.x, case.ids, case.gate_w)
    b = lay2.forward(case.x, case.ids, case.gate_w)
    assert torch.equal(a["Y_sum_gate"], b["Y_sum_gate"])


def test_full_size_outputs_are_finite_and_nonzero():
    case = get_case("qwen_t1")
    out = case.layer.forward(case.x, case.ids, case.gate_w)
    for proj in ("gate", "up"):
        y = out[f"Y_sum_{proj}"]
        assert torch.isfinite(y).all() and y.abs().max() > 0
