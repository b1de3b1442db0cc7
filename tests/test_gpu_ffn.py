"""The expert FFN after the gate/up projections -- SiLU(gate) * up, the dense fp16
down projection, the slot-order routed sum -- CUDA path against the oracle on the
same seeded inputs, within the outputs' 2e-3 bound (max relative error per output
vector, fp32 accumulation against fp64).

Two groups: the down step alone on seeded gate/up outputs (every shape and path:
the single-token kernel, the grouped multi-token kernels, column blocks, ragged
row counts, saturated SiLU, bad ids), and the whole FFN through the layer call on
the parity layers, the oracle running its own gate/up and down steps."""
import numpy as np
import pytest
import torch

from cases import SMALL, TOL, get_case, oracle_tokens, rel_err, x_bits
from mixed_precision_decode_b200 import bitsmoe as B
from mixed_precision_decode_b200 import synth
from mixed_precision_decode_b200.layer import SpectralMoEFFN

pytestmark = pytest.mark.gpu

# (name, d_model, d_ff, E, top_k, tokens, routing)
SHAPES = [
    ("tiny", 64, 32, 4, 2, (1, 4), "softmax_topk"),
    ("ragged", 37, 24, 6, 3, (1, 5), "softmax_topk"),
    ("min_dff", 40, 8, 3, 2, (1, 3), "softmax_topk"),
    ("wide_t1", 96, 8192, 8, 8, (1, 2), "softmax_topk"),   # top_k x d_ff too big for one CTA: grouped path at T = 1
    ("crowded", 256, 64, 4, 2, (48,), "softmax_topk"),     # ~24 tokens per expert: several tensor-core passes
    ("qwen", 2048, 768, 128, 8, (1, 8, 64), "uniform"),
    ("mixtral", 4096, 14336, 8, 2, (1, 16), "zipf"),
]


def _inputs(name, d_model, d_ff, E, K, T, routing, seed, g_scale=2.0, u_scale=1.0):
    cfg = synth.LayerConfig(name, d_model, d_ff, E, K, min(d_model, 64), T, ((1, 1.0),), routing=routing, seed=seed)
    dev = torch.device("cuda")
    gen = synth.make_generator(seed, dev)
    w = synth.make_down(cfg, gen, dev)
    yg = (torch.randn((T, K, d_ff), generator=gen, device=dev) * g_scale).contiguous()
    yu = (torch.randn((T, K, d_ff), generator=gen, device=dev) * u_scale).contiguous()
    ids, gw = synth.make_routing(cfg, gen, dev, T)
    return w, yg, yu, ids, gw


def _run(w, yg, yu, ids, gw):
    E, d_model, d_ff = w.shape
    T, K = ids.shape
    dims = B.ffn_dims(d_model, d_ff, E, K)
    n = B.ffn_down_workspace_bytes(dims, T)
    ws = torch.empty(max(n, 256), dtype=torch.uint8, device="cuda") if n else None
    out = torch.full((T, d_model), float("nan"), device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    B.ffn_down(dims, w, yg, yu, ids, gw, T, out, ws, n, st)
    return out, B.read_status(st)


def _oracle(orc, w, yg, yu, ids, gw, toks=None):
    """Oracle out for the given tokens, on a copy of just their experts' down matrices."""
    ids_h = ids.cpu().numpy()
    toks = list(range(ids_h.shape[0])) if toks is None else toks
    ids_h = ids_h[toks]
    ex = sorted(set(int(v) for v in ids_h.ravel() if 0 <= v < w.shape[0]))
    remap = {e: j for j, e in enumerate(ex)}
    rid = np.vectorize(lambda v: remap.get(int(v), -1), otypes=[np.int32])(ids_h) if ids_h.size else ids_h
    wsub = w[torch.as_tensor(ex, device=w.device, dtype=torch.long)].cpu().numpy().view(np.uint16) if ex else \
        np.zeros((1,) + tuple(w.shape[1:]), np.uint16)
    out, st = orc.ffn_down(yg.cpu().numpy()[toks].astype(np.float64), yu.cpu().numpy()[toks].astype(np.float64),
                           wsub, rid, gw.cpu().numpy()[toks])
    return out, st


def _sample(T):
    return list(range(T)) if T <= 8 else sorted({0, 1, T // 2, T - 2, T - 1})


@pytest.mark.parametrize("shape", SHAPES, ids=[s[0] for s in SHAPES])
def test_ffn_down_against_oracle(shape, orc):
    name, d_model, d_ff, E, K, tokens, routing = shape
    for i, T in enumerate(tokens):
        w, yg, yu, ids, gw = _inputs(name, d_model, d_ff, E, K, T, routing, seed=900 + 10 * i + len(name))
        out, st = _run(w, yg, yu, ids, gw)
        assert st == 0
        toks = _sample(T)
        ref, ost = _oracle(orc, w, yg, yu, ids, gw, toks)
        assert ost == 0
        assert rel_err(out.cpu().numpy()[toks], ref) <= TOL, (name, T)


def test_ffn_down_launch_counts():
    q = B.ffn_dims(2048, 768, 128, 8)
    assert B.ffn_down_launches(q, 0) == 0 and B.ffn_down_launches(q, 1) == 1 and B.ffn_down_launches(q, 8) == 3
    assert B.ffn_down_workspace_bytes(q, 1) == 0 and B.ffn_down_workspace_bytes(q, 8) > 8 * 8 * 2048 * 4
    wide = B.ffn_dims(96, 8192, 8, 8)
    assert B.ffn_down_launches(wide, 1) == 3 and B.ffn_down_workspace_bytes(wide, 1) > 0


@pytest.mark.parametrize("T", [1, 3])
def test_ffn_down_saturated_silu(T, orc):
    """|gate| up to ~100: SiLU saturates to v and to 0 (e^-v overflows to Inf)."""
    w, yg, yu, ids, gw = _inputs("sat", 64, 64, 4, 2, T, "softmax_topk", seed=950 + T, g_scale=30.0)
    out, st = _run(w, yg, yu, ids, gw)
    assert st == 0 and torch.isfinite(out).all()
    ref, _ = _oracle(orc, w, yg, yu, ids, gw)
    assert rel_err(out.cpu().numpy(), ref) <= TOL


@pytest.mark.parametrize("T", [1, 6])
def test_ffn_down_beyond_fp16_range(T, orc):
    """|h| up to ~1e7 (far past fp16's 65504): the grouped tensor-core kernel scales each
    token's h by a power of two before splitting it into fp16 parts."""
    w, yg, yu, ids, gw = _inputs("big", 128, 256, 4, 2, T, "softmax_topk", seed=955 + T, g_scale=3000.0,
                                 u_scale=1000.0)
    out, st = _run(w, yg, yu, ids, gw)
    assert st == 0 and torch.isfinite(out).all()
    ref, _ = _oracle(orc, w, yg, yu, ids, gw)
    assert rel_err(out.cpu().numpy(), ref) <= TOL


@pytest.mark.parametrize("T", [1, 3])
def test_ffn_down_bad_ids(T, orc):
    """A slot with an id outside [0, E) is left out of its token's sum and sets
    ST_BADEXPERT; the other slots are unaffected."""
    w, yg, yu, ids, gw = _inputs("bad", 48, 32, 5, 3, T, "softmax_topk", seed=960 + T)
    ids = ids.clone()
    ids[0, 1] = -1
    if T > 1:
        ids[T - 1, 0] = 5
    out, st = _run(w, yg, yu, ids, gw)
    assert st == B.ST_BADEXPERT
    ref, ost = _oracle(orc, w, yg, yu, ids, gw)
    assert ost == orc.ST_BADEXPERT
    assert rel_err(out.cpu().numpy(), ref) <= TOL


def test_ffn_down_empty_batch_writes_nothing():
    w, yg, yu, ids, gw = _inputs("empty", 32, 16, 2, 1, 1, "softmax_topk", seed=970)
    out = torch.full((1, 32), 7.0, device="cuda")
    B.ffn_down(B.ffn_dims(32, 16, 2, 1), w, yg, yu, ids, gw, 0, out)
    torch.cuda.synchronize()
    assert bool((out == 7.0).all())


def _ffn(case, seed):
    gen = synth.make_generator(seed, torch.device("cuda"))
    return SpectralMoEFFN(case.layer, synth.make_down(case.cfg, gen, torch.device("cuda")))


FFN_CASES = [n for n in SMALL if SMALL[n].d_out % 8 == 0] + ["qwen_t1", "qwen_t64", "mixtral_t16"]


def test_ffn_refuses_a_d_ff_not_multiple_of_8():
    """The down matrices' rows must stay 16-byte aligned: the ragged parity layer
    (d_out = 37) is refused on the host, before any launch, and nothing is written."""
    case = get_case("ragged")
    assert case.cfg.d_out % 8 != 0
    w = torch.zeros((case.cfg.n_experts, case.cfg.d_in, case.cfg.d_out), dtype=torch.float16, device="cuda")
    ffn = SpectralMoEFFN(case.layer, w)
    out = torch.full((case.cfg.tokens, case.cfg.d_in), 3.0, device="cuda")
    with pytest.raises(B.BitsMoEError) as ei:
        ffn.forward(case.x, case.ids, case.gate_w, out=out)
    assert ei.value.code == B.EINVAL
    torch.cuda.synchronize()
    assert bool((out == 3.0).all())


@pytest.mark.parametrize("name", FFN_CASES)
def test_ffn_end_to_end_against_oracle(name, orc):
    """The whole FFN through SpectralMoEFFN.forward (the layer call, then the down
    call in the same stream: on one token the down kernel's programmatic launch
    follows the fused layer kernel) against the oracle's gate/up from its own
    blobs followed by its down step."""
    case = get_case(name)
    ffn = _ffn(case, 4000 + len(name))
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = ffn.forward(case.x, case.ids, case.gate_w, status=st)
    assert B.read_status(st) == 0
    T = case.cfg.tokens
    if case.cfg.name in SMALL or T <= 4:
        toks = list(range(T))
    else:  # the sampling of the gate/up parity tests: the oracle's expert loops are slow at full size
        toks = [0, T // 3, T - 1] if case.cfg.d_out * case.cfg.rank < 4_000_000 else [0, T - 1]
    Ye = {}
    for proj in ("gate", "up"):
        Zref = orc.shared_proj(case.host[proj]["phi_t"], x_bits(case)[toks])
        Ye[proj], _ = oracle_tokens(case, orc, proj, toks, Zref)
    ids_h = case.ids.cpu().numpy()[toks]
    ex = sorted(set(int(v) for v in ids_h.ravel()))
    remap = {e: j for j, e in enumerate(ex)}
    rid = np.vectorize(remap.get, otypes=[np.int32])(ids_h)
    wsub = ffn.w_down[torch.as_tensor(ex, device="cuda")].cpu().numpy().view(np.uint16)
    ref, ost = orc.ffn_down(Ye["gate"], Ye["up"], wsub, rid, case.gate_w.cpu().numpy()[toks])
    assert ost == 0
    assert rel_err(out.cpu().numpy()[toks], ref) <= TOL


def test_ffn_repeated_single_token_calls_in_a_graph(orc):
    """Single-token FFN steps captured in one CUDA graph, layer and down kernels
    alternating with programmatic launches, replayed twice: every step matches a
    plain call."""
    case = get_case("tiny")
    ffn = _ffn(case, 4100)
    x, ids, gw = case.x[:1].contiguous(), case.ids[:1].contiguous(), case.gate_w[:1].contiguous()
    ref = ffn.forward(x, ids, gw).clone()
    outs = [torch.empty_like(ref) for _ in range(3)]
    ys = ffn.gate_up_buffers(1, x.device)  # buffers the graph reuses
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        ffn.forward(x, ids, gw, out=outs[0], gate_up=ys)  # warm-up on the capture stream
        torch.cuda.synchronize()
        with torch.cuda.graph(g, stream=s):
            for o in outs:
                ffn.forward(x, ids, gw, out=o, gate_up=ys)
    for _ in range(2):
        for o in outs:
            o.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        for o in outs:
            assert rel_err(o.cpu().numpy(), ref.cpu().numpy()) <= 1e-5


@pytest.mark.parametrize("name", ["tiny", "qwen_t1"])
def test_ffn_forward_equals_layer_then_down(name):
    """bitsmoe_ffn_forward (one call) gives what bitsmoe_layer_forward followed by
    bitsmoe_ffn_down gives, up to the order of the single-token layer kernel's fp32
    atomic additions (1e-5 of the vector maximum)."""
    case = get_case(name)
    ffn = _ffn(case, 4200)
    x, ids, gw = case.x[:1].contiguous(), case.ids[:1].contiguous(), case.gate_w[:1].contiguous()
    one = ffn.forward(x, ids, gw)
    ys = case.layer.forward(x, ids, gw, want_experts=True)
    two = torch.empty_like(one)
    n = B.ffn_down_workspace_bytes(ffn.dims, 1)
    ws = torch.empty(max(n, 256), dtype=torch.uint8, device="cuda")
    B.ffn_down(ffn.dims, ffn.w_down, ys["Y_experts_gate"], ys["Y_experts_up"], ids, gw, 1, two, ws, n)
    assert rel_err(one.cpu().numpy(), two.cpu().numpy()) <= 1e-5
