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
