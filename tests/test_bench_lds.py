"""The shared-memory bound bench.py reports for the multi-token path: the lookup
wavefront count on hand-computed cases, and the peak from unit counts."""
import numpy as np

import bench


class _Cfg:
    d_out = 64  # two 32-row tiles


def _counts(row):
    r = np.array(row, dtype=np.int64)
    return {"gate": r[None, :].repeat(3, 0), "up": r[None, :].repeat(3, 0)}


def test_one_token_uses_4_byte_lookups():
    # expert 1: 40 two-bit members -> 2 words of 32 members x 2 planes = 4 plane words;
    # 2 tiles; one token -> 8 wavefronts per (plane word, tile); both projections
    counts = _counts([0, 0, 0, 0, 0, 40, 0, 0])
    assert bench.lds_wavefronts(_Cfg, counts, np.array([[1]]), 1) == 2 * (4 * 2 * 8)


def test_token_groups_of_four_use_pairs():
    # five tokens on one expert -> groups of 4 (two pairs, 32 wavefronts) and 1 (8)
    counts = _counts([0, 0, 0, 0, 0, 40, 0, 0])
    ids = np.array([[1], [1], [1], [1], [1]])
    assert bench.lds_wavefronts(_Cfg, counts, ids, 5) == 2 * (4 * 2 * (32 + 8))
    # three tokens -> one group of 3: two pairs (the second half empty)
    assert bench.lds_wavefronts(_Cfg, counts, ids[:3], 3) == 2 * (4 * 2 * 32)


def test_fp16_and_zero_width_members_are_not_looked_up():
    # 10 fp16 members and 100 zero-width members only: no bit-plane words
    counts = _counts([10, 0, 0, 0, 0, 0, 0, 100])
    assert bench.lds_wavefronts(_Cfg, counts, np.array([[0], [2]]), 2) == 0


def test_every_width_group_counts_its_planes():
    # one member in each bit-plane group (8, 6, 4, 3, 2, 1): 24 plane words
    counts = _counts([0, 1, 1, 1, 1, 1, 1, 0])
    assert bench.lds_wavefronts(_Cfg, counts, np.array([[0]]), 1) == 2 * (24 * 2 * 8)


def test_lds_peak_from_unit_counts():
    assert abs(bench.lds_peak_gbs(1965.0, 148) - 128 * 148 * 1.965) < 1e-6


class _TinyOracleStep:
    """A layer step of the real oracle on tiny inputs (Phi^T x for 4 rows)."""

    def __init__(self):
        import oracle
        oracle.build()
        self.o = oracle
        rng = np.random.default_rng(3)
        self.phi = rng.standard_normal((4, 64)).astype(np.float16).view(np.uint16)
        self.x = rng.standard_normal((1, 64)).astype(np.float16).view(np.uint16)
        self.ref = self.o.shared_proj(self.phi, self.x)
        self.bad = 0

    def run(self, i):
        z = self.o.shared_proj(self.phi, self.x)
        if not np.array_equal(z, self.ref):
            self.bad += 1


def test_oracle_on_every_host_core_runs_independent_steps():
    s = _TinyOracleStep()
    el, n = bench.time_oracle_threads(s, 3, 0.3)
    assert el >= 0.3 and n >= 3 and s.bad == 0
    assert bench.host_cores() >= 1 and isinstance(bench.cpu_model(), str)
