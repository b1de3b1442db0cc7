"""The 48-layer Qwen3-30B-A3B-shaped stack (~2.08 bits, softmax top-8 routing)
at 8 and 32 decode tokens, against the oracle: sampled layers (the first and
the last seed of the stack), sampled tokens, and every expert routed to them.

At 8 tokens a layer routes ~1.2 tokens per touched expert, so most experts run
the multi-token kernel's one-token branch; the last case routes 64 distinct
experts (every touched expert gets exactly one token), which forces that
branch for every expert of the call."""
import numpy as np
import pytest
import torch

from cases import TOL, Case, oracle_tokens, rel_err, x_bits
from mixed_precision_decode_b200 import bitsmoe as B
from mixed_precision_decode_b200 import synth

pytestmark = pytest.mark.gpu

STACK = synth.CONFIGS["qwen_stack"]
_cache = {}


def _case(T: int, layer: int) -> Case:
    key = (T, layer)
    if key not in _cache:
        _cache.clear()  # one full-size layer on the device at a time
        cfg = synth.scaled(STACK, name=f"qwen_stack_t{T}_l{layer}", tokens=T, seed=STACK.seed + layer)
        _cache[key] = Case(cfg)
    return _cache[key]


def _check(case, orc, ids, gw, toks):
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = case.layer.forward(case.x, ids, gw, want_experts=True, want_z=True, status=st)
    assert B.read_status(st) == 0
    for proj in ("gate", "up"):
        Zref = orc.shared_proj(case.host[proj]["phi_t"], x_bits(case))
        assert rel_err(out[f"Z_{proj}"].cpu().numpy(), Zref) <= TOL
        Ye_ref, Ys_ref = oracle_tokens(case, orc, proj, toks, Zref[toks], ids=ids, gate_w=gw)
        assert rel_err(out[f"Y_experts_{proj}"].cpu().numpy()[toks], Ye_ref) <= TOL
        assert rel_err(out[f"Y_sum_{proj}"].cpu().numpy()[toks], Ys_ref) <= TOL


@pytest.mark.parametrize("T,layer", [(8, 0), (8, 47), (32, 0), (32, 47)])
def test_stack_layer_against_oracle(T, layer, orc):
    case = _case(T, layer)
    assert B.layer_launches(case.proj["gate"].plan, case.proj["up"].plan, T) > 1  # the multi-token path
    toks = [0, T // 2, T - 1]
    _check(case, orc, case.ids, case.gate_w, toks)


def test_stack_t8_every_expert_one_token(orc):
    case = _case(8, 0)
    gen = torch.Generator(device="cuda").manual_seed(4242)
    ids = torch.randperm(STACK.n_experts, generator=gen, device="cuda")[:8 * STACK.top_k]
    ids = ids.reshape(8, STACK.top_k).to(torch.int32).contiguous()
    gw = torch.softmax(torch.randn((8, STACK.top_k), generator=gen, device="cuda"), dim=1).contiguous()
    assert len(set(ids.cpu().numpy().ravel().tolist())) == 8 * STACK.top_k
    _check(case, orc, ids, gw, list(range(8)))
