"""The offline step on the GPU -- shared-basis spectral decomposition, widths by
descending amplitude, packing -- against the oracle and the definitions.

The decomposition is unique only up to the sign of each pair (phi_k, p_{e,k}), and
for singular values that nearly coincide only up to a rotation of their vectors.
So: on a matrix with well-separated singular values, Phi, a and p are compared
with the oracle's (numpy SVD) after the same sign rule; on random matrices (a
clustered spectrum) the singular values are compared with the oracle's and the
rest is checked for validity -- Phi orthonormal, p unit, and the factors
reconstructing every W_e.  End to end, decomposition + packing at width 16 +
the decode path give W_e x within the outputs' 2e-3 bound."""
import numpy as np
import pytest
import torch

from cases import TOL, rel_err
from mixed_precision_decode_b200 import bitsmoe as B
from mixed_precision_decode_b200 import synth
from mixed_precision_decode_b200.layer import PackedProjection, SpectralMoELayer, decompose_and_pack, fqcm_widths

pytestmark = pytest.mark.gpu


def _decompose(W, r):
    E, d_out, d_in = W.shape
    n = B.ssd_workspace_bytes(E, d_out, d_in, r)
    assert n > 0
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    out = {"phi_t": torch.empty((r, d_in), dtype=torch.float16, device="cuda"),
           "phi_t32": torch.empty((r, d_in), dtype=torch.float32, device="cuda"),
           "sigma": torch.empty(r, dtype=torch.float32, device="cuda"),
           "amps": torch.empty((E, r), dtype=torch.float32, device="cuda"),
           "comps": torch.empty((E, r, d_out), dtype=torch.float32, device="cuda")}
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    B.ssd_decompose(W, r, out["phi_t"], out["amps"], out["comps"], ws, n, sigma=out["sigma"],
                    phi_t32=out["phi_t32"], status=st)
    assert B.read_status(st) == 0
    return {k: v.cpu().numpy() for k, v in out.items()}


def _sign_fix(Phi, p):
    """The library's sign rule on the oracle's factors: each phi_k's entry of largest
    magnitude (the first on a tie) positive, p_{e,k} flipped with it."""
    idx = np.argmax(np.abs(Phi), axis=0)
    sgn = np.where(Phi[idx, np.arange(Phi.shape[1])] < 0, -1.0, 1.0)
    return Phi * sgn, p * sgn[None, :, None]


def _separated(E, d_out, d_in, seed):
    """W_cat = U diag(s) V^T with s geometric from 10 to 2: the smallest gap between
    squared singular values is ~0.2 of the largest 100, so fp32 eigenvectors of the
    Gram matrix carry errors of order 6e-8 x 100 / 0.2 = 3e-5 (the tolerances below)."""
    g = torch.Generator().manual_seed(seed)
    U, _ = torch.linalg.qr(torch.randn(E * d_out, d_in, generator=g, dtype=torch.float64))
    V, _ = torch.linalg.qr(torch.randn(d_in, d_in, generator=g, dtype=torch.float64))
    s = 10.0 * (0.2 ** (torch.arange(d_in, dtype=torch.float64) / (d_in - 1)))
    return ((U * s) @ V.T).reshape(E, d_out, d_in).numpy()


@pytest.mark.parametrize("r", [64, 40])
def test_ssd_matches_oracle_on_separated_spectrum(r, orc):
    E, d_out, d_in = 4, 32, 64
    W = _separated(E, d_out, d_in, 11)
    g = _decompose(torch.from_numpy(W).float().cuda().contiguous(), r)
    Phi, a, p = orc.ssd_decompose(W, r)
    Phi, p = _sign_fix(Phi, p)
    s_ref = np.sqrt((a ** 2).sum(axis=0))  # ||P[:, k]|| = s_k
    assert np.allclose(g["sigma"], s_ref, rtol=1e-4, atol=0)
    assert np.max(np.abs(g["phi_t32"].T - Phi)) <= 2e-4
    assert np.max(np.abs(g["phi_t"].astype(np.float64).T - Phi)) <= 1e-3  # the fp16 copy
    assert np.max(np.abs(g["amps"] - a)) <= 2e-4 * a.max()
    assert np.max(np.abs(g["comps"] - p)) <= 5e-4


@pytest.mark.parametrize("E,d_out,d_in", [(8, 96, 128), (3, 8, 40)])
def test_ssd_invariants_on_random_matrices(E, d_out, d_in, orc):
    """(3, 8, 40) is rank-deficient (24 stacked rows < 40 columns): its last 16
    singular values are 0, their directions arbitrary; they must still complete the
    basis and reconstruct W exactly."""
    rng = np.random.default_rng(21 + d_in)
    W = rng.standard_normal((E, d_out, d_in)) / np.sqrt(d_in)
    r = d_in
    nz = min(r, E * d_out)  # singular values that are not 0
    g = _decompose(torch.from_numpy(W).float().cuda().contiguous(), r)
    _, a, _ = orc.ssd_decompose(W, nz)  # the oracle's SVD has min(rows, d_in) directions
    s_ref = np.sqrt((a ** 2).sum(axis=0))
    assert np.all(np.diff(g["sigma"]) <= 1e-6 * g["sigma"][0])
    assert np.allclose(g["sigma"][:nz], s_ref[:nz], rtol=1e-4, atol=0)
    assert np.all(g["sigma"][nz:] <= 1e-3 * s_ref[0])
    Phi = g["phi_t32"].astype(np.float64).T
    assert np.max(np.abs(Phi.T @ Phi - np.eye(r))) <= 2e-5
    pn = np.linalg.norm(g["comps"][:, :nz].astype(np.float64), axis=2)
    assert np.max(np.abs(pn - 1.0)) <= 1e-5
    assert np.all(g["amps"] >= 0)
    for e in range(E):
        rec = (g["comps"][e].astype(np.float64).T * g["amps"][e]) @ Phi.T  # sum_k a p phi^T
        assert np.linalg.norm(rec - W[e]) <= 1e-4 * np.linalg.norm(W[e])
    # the sign rule
    idx = np.argmax(np.abs(Phi), axis=0)
    assert np.all(Phi[idx, np.arange(r)] > 0)


def test_ssd_full_size_qwen_projection(orc):
    """A Qwen3-30B-A3B-shaped projection (128 experts of 768 x 2048, rank 2048):
    Phi orthonormal, p unit, the singular values descending and equal to the square
    roots of the fp64 eigenvalues of W_cat^T W_cat, two experts reconstructed."""
    E, d_out, d_in = 128, 768, 2048
    g = torch.Generator(device="cuda").manual_seed(31)
    W = (torch.randn((E, d_out, d_in), generator=g, device="cuda") / d_in ** 0.5).contiguous()
    out = _decompose(W, d_in)
    Phi = out["phi_t32"].astype(np.float64).T
    assert np.max(np.abs(Phi.T @ Phi - np.eye(d_in))) <= 1e-4  # fp32 eigensolver, n = 2048
    assert np.max(np.abs(np.linalg.norm(out["comps"][[0, E - 1]].astype(np.float64), axis=2) - 1.0)) <= 1e-5
    assert np.all(np.diff(out["sigma"]) <= 1e-6 * out["sigma"][0])
    Wh = W.cpu().numpy().astype(np.float64)
    A = Wh.reshape(E * d_out, d_in)
    G = A.T @ A  # W_cat^T W_cat, fp64
    lam = np.linalg.eigvalsh(G)[::-1]
    s_ref = np.sqrt(np.maximum(lam, 0))
    assert np.allclose(out["sigma"], s_ref, rtol=2e-4, atol=1e-4 * s_ref[0])
    for e in (0, E - 1):
        rec = (out["comps"][e].astype(np.float64).T * out["amps"][e]) @ Phi.T
        assert np.linalg.norm(rec - Wh[e]) <= 2e-4 * np.linalg.norm(Wh[e])


def test_decompose_pack_decode_all_16_bit():
    """Decomposition, widths all 16, packing and the decode path reproduce W_e x
    (the definition, fp64) within 2e-3 for every routed slot."""
    E, d_out, d_in, K, T = 4, 32, 64, 2, 5
    rng = np.random.default_rng(41)
    Wg = rng.standard_normal((E, d_out, d_in)) / np.sqrt(d_in)
    Wu = rng.standard_normal((E, d_out, d_in)) / np.sqrt(d_in)
    pg, _ = decompose_and_pack(torch.from_numpy(Wg).float().cuda(), d_in, (16,), (d_in,), K)
    pu, _ = decompose_and_pack(torch.from_numpy(Wu).float().cuda(), d_in, (16,), (d_in,), K)
    layer = SpectralMoELayer(pg, pu)
    cfg = synth.LayerConfig("ssd_e2e", d_in, d_out, E, K, d_in, T, ((16, 1.0),), seed=42)
    gen = synth.make_generator(42, torch.device("cuda"))
    x = torch.randn((T, d_in), generator=gen, device="cuda").to(torch.float16)
    ids, gw = synth.make_routing(cfg, gen, torch.device("cuda"), T)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = layer.forward(x, ids, gw, want_experts=True, status=st)
    assert B.read_status(st) == 0
    X = x.cpu().numpy().astype(np.float64)
    idh = ids.cpu().numpy()
    for name, Wm in (("gate", Wg), ("up", Wu)):
        ref = np.stack([np.stack([Wm[idh[t, j]] @ X[t] for j in range(K)]) for t in range(T)])
        assert rel_err(out[f"Y_experts_{name}"].cpu().numpy(), ref) <= TOL


def test_decompose_pack_widths_follow_amplitudes():
    """The widths the pipeline packs follow its amplitudes (a larger a never gets a
    width listed later; equal a: lower k first), with the given counts, and the
    packed blob holds exactly those counts per expert."""
    E, d_out, d_in = 3, 16, 48
    rng = np.random.default_rng(51)
    W = rng.standard_normal((E, d_out, d_in))
    order, counts = (8, 4, 2, 1, 0), (4, 8, 16, 12, 8)
    pk, dec = decompose_and_pack(torch.from_numpy(W).float().cuda(), d_in, order, counts, 2)
    w = dec["widths"].numpy()
    a = dec["amps"].cpu().numpy()
    rank = {b: i for i, b in enumerate(order)}
    for e in range(E):
        assert [int((w[e] == b).sum()) for b in order] == list(counts)
        seq = sorted(range(d_in), key=lambda k: (-a[e, k], k))
        assert [rank[int(w[e, k])] for k in seq] == sorted(rank[int(w[e, k])] for k in seq)
    h = pk.plan.header()
    for e in range(E):
        n = h[64 + 64 * e + 44: 64 + 64 * e + 60].view(np.uint16)  # counts in width order 16,8,6,4,3,2,1,0
        assert [int(n[1]), int(n[3]), int(n[5]), int(n[6]), int(n[7])] == list(counts)


def test_fqcm_allocation_pipeline():
    """Decomposition, the FQCM allocation from seeded calibration tokens (z on the
    GPU), packing and decoding: the budget holds, every width is in the set, and on
    its own cost the allocation is no worse than the fixed-fraction rule at the same
    average bits (which it is free to choose), nor than uniform 2 bits."""
    E, d_out, d_in, K, Tc = 6, 64, 128, 2, 256
    rng = np.random.default_rng(61)
    W = torch.from_numpy(rng.standard_normal((E, d_out, d_in)) / np.sqrt(d_in)).float().cuda()
    order, counts = (8, 4, 3, 2, 1, 0), (3, 10, 26, 51, 25, 13)
    _, dec = decompose_and_pack(W, d_in, order, counts, K)
    cfg = synth.LayerConfig("fqcm", d_in, d_out, E, K, d_in, Tc, ((2, 1.0),), seed=62)
    gen = synth.make_generator(62, torch.device("cuda"))
    xc = torch.randn((Tc, d_in), generator=gen, device="cuda").to(torch.float16)
    ids, gw = synth.make_routing(cfg, gen, torch.device("cuda"), Tc)
    avg = sum(b * c for b, c in zip(order, counts)) / d_in
    widths, loss, parts = fqcm_widths(dec, xc, ids, gw, avg)
    w = widths.numpy()
    assert set(np.unique(w).tolist()) <= set(B.WIDTH_SET)
    assert int(d_out * w.astype(np.int64).sum()) <= int(avg * E * d_in * d_out)
    a = dec["amps"].cpu().numpy().astype(np.float64)
    idx = {b: i for i, b in enumerate(B.WIDTH_SET)}
    def cost(ws):
        wi = np.vectorize(idx.get)(ws)
        return float((a ** 2 * parts["beta"] * np.take_along_axis(parts["eps"], wi[..., None], 2)[..., 0]).sum())
    assert abs(cost(w) - loss) <= 1e-9 * max(loss, 1.0)
    # the relaxation's optimum is below both; the allocation stops at the first step that
    # does not fit, so it can exceed that optimum by at most one step's saving (1 % here)
    assert loss <= cost(dec["widths"].numpy()) * 1.01
    assert loss <= cost(np.full_like(w, 2)) * 1.01
    pk = PackedProjection.from_factors(dec["phi_t"], dec["amps"], dec["comps"], widths, K)
    layer = SpectralMoELayer(pk, pk)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = layer.forward(xc[:3], ids[:3], gw[:3], status=st)
    assert B.read_status(st) == 0 and torch.isfinite(out["Y_sum_gate"]).all()
