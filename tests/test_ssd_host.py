"""Host side of the offline step (CPU): the library's width assignment against the
oracle's on seeded amplitudes, bit-exact, and the decomposition's argument checks,
which run before any device work."""
import numpy as np
import pytest


@pytest.fixture(scope="module")
def B():
    from mixed_precision_decode_b200 import build
    build.build()
    from mixed_precision_decode_b200 import bitsmoe
    return bitsmoe


@pytest.mark.parametrize("seed,E,r", [(1, 4, 64), (2, 3, 2048), (3, 1, 7)])
def test_assign_widths_matches_oracle(B, orc, seed, E, r):
    rng = np.random.default_rng(seed)
    a = rng.lognormal(0, 0.5, (E, r)).astype(np.float32)
    a[:, ::5] = a[:, 1:2]  # ties
    order = (16, 8, 4, 3, 2, 1, 0)
    cuts = np.sort(rng.integers(0, r + 1, len(order) - 1))
    counts = np.diff(np.concatenate([[0], cuts, [r]])).astype(np.int32)
    assert np.array_equal(B.assign_widths(a, order, counts), orc.assign_widths(a, order, counts))


def test_assign_widths_errors(B):
    a = np.ones((2, 4), np.float32)
    with pytest.raises(B.BitsMoEError) as ei:
        B.assign_widths(a, (8, 0), (2, 1))  # counts sum to 3, not 4
    assert ei.value.code == B.EINVAL
    with pytest.raises(B.BitsMoEError) as ei:
        B.assign_widths(a, (5, 0), (2, 2))  # 5 bits is not a width
    assert ei.value.code == B.EWIDTH


def test_ssd_argument_checks(B):
    L = B.lib()
    assert B.ssd_workspace_bytes(4, 32, 64, 65) == 0  # rank > d_in
    assert B.ssd_workspace_bytes(0, 32, 64, 64) == 0
    args = (256, 256, 256, 256, 256, 256, 1 << 20, None, None)
    assert L.bitsmoe_ssd_decompose(256, 4, 32, 64, 65, *args) == B.EINVAL
    assert L.bitsmoe_ssd_decompose(None, 4, 32, 64, 64, *args) == B.EINVAL
    assert L.bitsmoe_ssd_decompose(256, 4, 32, 64, 64, 256, None, None, 256, 256, 0x1010, 1 << 20, None,
                                   None) == B.EINVAL  # workspace not 256-byte aligned


# --------------------------------------------------------------------------
# FQCM and the bit-budget allocation: the library against the oracle, bit-exact
# --------------------------------------------------------------------------

def _unit(rng, E, r, d_out):
    p = rng.standard_normal((E, r, d_out)).astype(np.float32)
    return p / np.linalg.norm(p, axis=2, keepdims=True)


@pytest.mark.parametrize("seed,E,r,d_out", [(1, 3, 40, 37), (2, 2, 64, 768)])
def test_fqcm_eps_matches_oracle(B, orc, seed, E, r, d_out):
    """Unit directions plus the special cases: a zero direction, a non-unit one past
    fp16's scale range, one with a NaN."""
    rng = np.random.default_rng(seed)
    p = _unit(rng, E, r, d_out)
    p[0, 0] = 0.0
    p[0, 1] *= 1e6
    p[0, 2, 3] = np.nan
    got, ref = B.fqcm_eps(p), orc.fqcm_eps(p)
    assert np.array_equal(got, ref, equal_nan=True)


def test_fqcm_beta_matches_oracle(B, orc):
    rng = np.random.default_rng(3)
    T, K, E, r = 50, 4, 6, 33
    Z = rng.standard_normal((T, r)).astype(np.float32)
    ids = rng.integers(-1, E + 1, (T, K)).astype(np.int32)  # some ids out of range
    g = rng.uniform(0, 1, (T, K)).astype(np.float32)
    assert np.array_equal(B.fqcm_beta(Z, ids, g, E), orc.fqcm_beta(Z, ids, g, E))


@pytest.mark.parametrize("seed", [4, 5])
def test_allocate_widths_matches_oracle(B, orc, seed):
    """The same inputs (seeded amplitudes, importances and distortions from the
    oracle's own eps), several budgets from none to everything: identical widths
    and total cost."""
    rng = np.random.default_rng(seed)
    E, r, d_out = 3, 50, 24
    a = rng.lognormal(0, 0.5, (E, r)).astype(np.float32)
    beta = rng.lognormal(0, 1.0, (E, r))
    beta[0, :3] = 0.0
    eps = orc.fqcm_eps(_unit(rng, E, r, d_out))
    eps[1, 4, 2] = np.nan  # a component without a finite cost
    for avg in (0.0, 0.5, 2.08, 3.0, 16.0):
        budget = int(avg * E * r * d_out)
        w, loss = B.allocate_widths(a, beta, eps, d_out, budget)
        w_ref, loss_ref = orc.allocate_widths(a, beta, eps, d_out, budget)
        assert np.array_equal(w, w_ref) and loss == loss_ref, avg
        assert int(d_out * w.astype(np.int64).sum()) <= budget
        assert w[1, 4] == 0


def test_fqcm_argument_checks(B):
    L = B.lib()
    assert L.bitsmoe_fqcm_eps(None, 1, 1, 1, None) == B.EINVAL
    assert L.bitsmoe_fqcm_beta(None, None, None, 1, 1, 1, 1, 256) == B.EINVAL
    beta = np.full((1, 1), 7.0)
    assert L.bitsmoe_fqcm_beta(None, None, None, 0, 1, 1, 1, beta.ctypes.data) == B.OK  # no tokens: zeros
    assert beta[0, 0] == 0.0
    assert L.bitsmoe_allocate_widths(None, None, None, 1, 1, 1, 0, None, None) == B.EINVAL


# --------------------------------------------------------------------------
# property tests over random shapes, ties and budgets (bounded example counts)
# --------------------------------------------------------------------------
from hypothesis import HealthCheck, given, settings  # noqa: E402
from hypothesis import strategies as st  # noqa: E402


@settings(max_examples=40, deadline=None, suppress_health_check=[HealthCheck.function_scoped_fixture])
@given(E=st.integers(1, 4), r=st.integers(1, 24), seed=st.integers(0, 2 ** 31 - 1),
       levels=st.integers(1, 6))
def test_assign_widths_property(B, orc, E, r, seed, levels):
    rng = np.random.default_rng(seed)
    a = rng.integers(0, levels, (E, r)).astype(np.float32)  # few distinct values: many ties
    order = tuple(int(b) for b in rng.permutation([0, 1, 2, 3, 4, 6, 8, 16])[:rng.integers(1, 9)])
    cuts = np.sort(rng.integers(0, r + 1, len(order) - 1))
    counts = np.diff(np.concatenate([[0], cuts, [r]])).astype(np.int32)
    assert np.array_equal(B.assign_widths(a, order, counts), orc.assign_widths(a, order, counts))


@settings(max_examples=40, deadline=None, suppress_health_check=[HealthCheck.function_scoped_fixture])
@given(E=st.integers(1, 3), r=st.integers(1, 20), d_out=st.integers(1, 40), seed=st.integers(0, 2 ** 31 - 1),
       frac=st.floats(0.0, 1.2))
def test_fqcm_and_allocation_property(B, orc, E, r, d_out, seed, frac):
    rng = np.random.default_rng(seed)
    p = rng.standard_normal((E, r, d_out)).astype(np.float32)
    p[rng.random((E, r)) < 0.1] = 0.0  # some zero directions
    eps = B.fqcm_eps(p)
    assert np.array_equal(eps, orc.fqcm_eps(p), equal_nan=True)
    a = rng.lognormal(0, 1, (E, r)).astype(np.float32)
    beta = rng.lognormal(0, 1, (E, r)) * (rng.random((E, r)) > 0.2)
    budget = int(frac * 16 * E * r * d_out)
    w, loss = B.allocate_widths(a, beta, eps, d_out, budget)
    w_ref, loss_ref = orc.allocate_widths(a, beta, eps, d_out, budget)
    assert np.array_equal(w, w_ref) and loss == loss_ref
    assert int(d_out * w.astype(np.int64).sum()) <= budget
