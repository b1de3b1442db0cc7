"""The fused single-token layer path (one persistent launch for both
projections) against the oracle and against the general multi-kernel path."""
import numpy as np
import pytest
import torch

from cases import TOL, get_case, oracle_tokens, rel_err, x_bits
from mixed_precision_decode_b200 import bitsmoe as B

pytestmark = pytest.mark.gpu


def _one(case, t, ids=None, gw=None, **kw):
    ids = case.ids if ids is None else ids
    gw = case.gate_w if gw is None else gw
    return case.layer.forward(case.x[t:t + 1].contiguous(), ids[t:t + 1].contiguous(), gw[t:t + 1].contiguous(), **kw)


def _general(case, t, ids=None, gw=None):
    """Same token through the general kernels (shared projection + expert call)."""
    ids = case.ids if ids is None else ids
    gw = case.gate_w if gw is None else gw
    out = {}
    for proj in ("gate", "up"):
        pk = case.proj[proj]
        r, K, d_out = pk.rank, pk.top_k, pk.d_out
        Z = torch.empty((1, r), dtype=torch.float32, device="cuda")
        B.shared_proj(pk.phi_t, case.x[t:t + 1].contiguous(), Z, 1, pk.d_in, r)
        Ye = torch.empty((1, K, d_out), dtype=torch.float32, device="cuda")
        Ys = torch.empty((1, d_out), dtype=torch.float32, device="cuda")
        n = B.expert_workspace_bytes(pk.plan, 1)
        ws = torch.empty(n, dtype=torch.uint8, device="cuda")
        B.expert_forward(pk.plan, pk.blob, Z, ids[t:t + 1].contiguous(), gw[t:t + 1].contiguous(), 1, Ye, Ys, ws, n)
        out[f"Y_sum_{proj}"], out[f"Y_experts_{proj}"], out[f"Z_{proj}"] = Ys, Ye, Z
    return out


@pytest.mark.parametrize("name", ["tiny", "ragged", "one_expert", "qwen_t1", "qwen_t64"])
def test_fused_t1_against_oracle(name, orc):
    case = get_case(name)
    assert B.layer_launches(case.proj["gate"].plan, case.proj["up"].plan, 1) == 1
    for t in sorted({0, case.cfg.tokens - 1}):
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        out = _one(case, t, want_experts=True, want_z=True, status=st)
        assert B.read_status(st) == 0
        for proj in ("gate", "up"):
            Zref = orc.shared_proj(case.host[proj]["phi_t"], x_bits(case)[t:t + 1])
            assert rel_err(out[f"Z_{proj}"].cpu().numpy(), Zref) <= TOL
            Ye_ref, Ys_ref = oracle_tokens(case, orc, proj, [t], Zref)
            assert rel_err(out[f"Y_experts_{proj}"].cpu().numpy(), Ye_ref) <= TOL
            assert rel_err(out[f"Y_sum_{proj}"].cpu().numpy(), Ys_ref) <= TOL


def test_fused_t1_repeated_calls_interleaved_with_batches():
    """Many single-token calls on one workspace (its counter and tagged z rows
    carry over from call to call), interleaved with batched calls, all agree
    with the general kernels to fp32 rounding."""
    case = get_case("qwen_t64")
    lay = case.layer
    gen = torch.Generator(device="cuda").manual_seed(5)
    for it in range(60):
        t = it % case.cfg.tokens
        ids = torch.randint(0, case.cfg.n_experts, case.ids.shape, generator=gen, device="cuda", dtype=torch.int32)
        out = _one(case, t, ids=ids, want_experts=True)
        ref = _general(case, t, ids=ids)
        for proj in ("gate", "up"):
            assert rel_err(out[f"Y_experts_{proj}"].cpu().numpy(), ref[f"Y_experts_{proj}"].cpu().numpy()) <= 1e-5
            assert rel_err(out[f"Y_sum_{proj}"].cpu().numpy(), ref[f"Y_sum_{proj}"].cpu().numpy()) <= 1e-5
        if it % 7 == 3:
            lay.forward(case.x[:5].contiguous(), case.ids[:5].contiguous(), case.gate_w[:5].contiguous())
    # the same call twice agrees to fp32 rounding: the routed sum is accumulated
    # with atomic adds, whose order may differ between runs.  Each element sums
    # ~80 partials (8 slots x ~10 CTAs); fp32 summation in any order is within
    # (n-1) * 2^-24 * sum|partials|, about 1e-5 of the vector's largest entry here.
    a = _one(case, 3)
    b = _one(case, 3)
    for proj in ("gate", "up"):
        assert rel_err(a[f"Y_sum_{proj}"].cpu().numpy(), b[f"Y_sum_{proj}"].cpu().numpy()) <= 1e-5


def test_fused_t1_workspace_shared_with_batches_across_tag_wrap():
    """One workspace shared by single-token and 5-token calls (the batched path
    writes its scratch after the fused path's persistent state), with the launch
    counter started just below the point where the 32-bit launch tag wraps: every
    single-token result matches the general kernels, and the counter advances by
    exactly one grid per single-token launch."""
    case = get_case("qwen_t64")
    pg, pu = case.proj["gate"], case.proj["up"]
    G = torch.cuda.get_device_properties(0).multi_processor_count
    n = max(B.layer_workspace_bytes(pg.plan, pu.plan, T) for T in (1, 5))
    ws = torch.zeros(n, dtype=torch.uint8, device="cuda")
    start = G * (2 ** 32 - 3)  # tags of the next launches: 2^32 - 2, 2^32 - 1, 1, 2, ...
    ws[:8].view(torch.int64)[0] = start
    d_out = case.cfg.d_out
    n_t1 = 0
    for it in range(8):
        t = it % case.cfg.tokens
        out = {k: torch.full((1, d_out), float("nan"), device="cuda") for k in ("Y_sum_gate", "Y_sum_up")}
        ios = [B.proj_io(p.plan, p.blob, p.phi_t, out[f"Y_sum_{name}"]) for name, p in (("gate", pg), ("up", pu))]
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        B.layer_forward(ios[0], ios[1], case.x[t:t + 1].contiguous(), case.ids[t:t + 1].contiguous(),
                        case.gate_w[t:t + 1].contiguous(), 1, ws, n, st)
        assert B.read_status(st) == 0
        n_t1 += 1
        ref = _general(case, t)
        for proj in ("gate", "up"):
            assert rel_err(out[f"Y_sum_{proj}"].cpu().numpy(), ref[f"Y_sum_{proj}"].cpu().numpy()) <= 1e-5, (it, proj)
        if it % 2 == 1:  # a batched call over the same workspace
            outb = {k: torch.empty((5, d_out), device="cuda") for k in ("Y_sum_gate", "Y_sum_up")}
            iob = [B.proj_io(p.plan, p.blob, p.phi_t, outb[f"Y_sum_{name}"]) for name, p in (("gate", pg), ("up", pu))]
            B.layer_forward(iob[0], iob[1], case.x[:5].contiguous(), case.ids[:5].contiguous(),
                            case.gate_w[:5].contiguous(), 5, ws, n, st)
            assert B.read_status(st) == 0
    torch.cuda.synchronize()
    assert int(ws[:8].view(torch.int64)[0]) == start + n_t1 * G


def test_fused_t1_bad_expert_id():
    case = get_case("qwen_t1")
    ids = case.ids.clone()
    ids[0, 2] = -5
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = _one(case, 0, ids=ids, want_experts=True, status=st)
    assert B.read_status(st) & B.ST_BADEXPERT
    ref = _general(case, 0, ids=ids)
    for proj in ("gate", "up"):
        assert torch.all(out[f"Y_experts_{proj}"][0, 2] == 0)
        assert rel_err(out[f"Y_sum_{proj}"].cpu().numpy(), ref[f"Y_sum_{proj}"].cpu().numpy()) <= 1e-5
    good = _one(case, 0)  # the workspace is still consistent after the bad call
    ref = _general(case, 0)
    assert rel_err(good["Y_sum_gate"].cpu().numpy(), ref["Y_sum_gate"].cpu().numpy()) <= 1e-5


def test_fused_t1_in_cuda_graph():
    case = get_case("qwen_t1")
    lay = case.layer
    x = case.x[0:1].clone()
    outs = [{k: torch.empty((1, case.cfg.d_out), dtype=torch.float32, device="cuda") for k in ("Y_sum_gate", "Y_sum_up")}
            for _ in range(6)]
    lay.forward(x, case.ids, case.gate_w, out=outs[0])
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for o in outs:
            lay.forward(x, case.ids, case.gate_w, out=o)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    ref = _general(case, 0)
    for o in outs:
        for proj in ("gate", "up"):
            assert rel_err(o[f"Y_sum_{proj}"].cpu().numpy(), ref[f"Y_sum_{proj}"].cpu().numpy()) <= 1e-5


def test_chained_call_prefetch_changes_nothing(orc):
    """A decode loop that names the next layer (its Phi^T is prefetched into L2)
    gets the same outputs as the plain call, at one token and at several."""
    case = get_case("qwen_t1")
    lay = case.layer
    for T in (1, 3):
        x, ids, gw = case.x[:T].contiguous(), case.ids[:T].contiguous(), case.gate_w[:T].contiguous()
        a = lay.forward(x, ids, gw, want_experts=True)
        b = lay.forward(x, ids, gw, want_experts=True, next_layer=lay)
        for k in a:  # two runs of the atomic routed sum: the fp32 summation-order bound (~1e-5)
            assert rel_err(a[k].cpu().numpy(), b[k].cpu().numpy()) <= 1e-5, (T, k)
