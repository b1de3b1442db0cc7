"""Pins of the oracle against things other than itself (CPU only).

Each test says what it pins and to what: a hand-derived golden blob, a
closed form, a library routine (numpy float16, LAPACK SVD, numpy matmul),
an invariant, or brute force on tiny inputs.
"""
import json
import os

import numpy as np
import pytest

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# --------------------------------------------------------------------------
# fp16 conversion: exhaustive against numpy's float16 (a library routine)
# --------------------------------------------------------------------------

def test_f16_to_f64_all_patterns(orc):
    h = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = orc.f16_bits_to_f64(h)
    ref = h.view(np.float16).astype(np.float64)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])
    # signed zeros keep their sign
    assert np.array_equal(np.signbit(ours[~nan]), np.signbit(ref[~nan]))


def _f32_cases():
    h = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    vals = h.view(np.float16).astype(np.float64)
    fin = np.sort(np.unique(vals[np.isfinite(vals)]))
    mids = (fin[:-1] + fin[1:]) / 2.0  # exact in fp64; ties for the converter
    mids32 = mids.astype(np.float32)
    up = np.nextafter(mids32, np.float32(np.inf))
    dn = np.nextafter(mids32, np.float32(-np.inf))
    rng = np.random.default_rng(123)
    rnd = (rng.standard_normal(20000) * np.exp2(rng.integers(-30, 20, 20000))).astype(np.float32)
    special = np.array([0.0, -0.0, np.inf, -np.inf, 65504, 65519.996, 65520, 65536, 1e-8, 2.0 ** -25,
                        2.0 ** -25 * 1.0000001, 2.0 ** -24, 3 * 2.0 ** -26, 1e-45, -1e-45, 1e30],
                       dtype=np.float32)
    return np.concatenate([fin.astype(np.float32), mids32, up, dn, rnd, special])


def test_f32_to_f16_against_numpy(orc):
    x = _f32_cases()
    ours = orc.f32_to_f16_bits(x)
    with np.errstate(over="ignore"):
        ref = x.astype(np.float16).view(np.uint16)
    assert np.array_equal(ours, ref), np.flatnonzero(ours != ref)[:10]


def test_f32_to_f16_nan_is_quiet_nan(orc):
    out = orc.f32_to_f16_bits(np.array([np.nan, -np.nan], np.float32))
    assert (out[0] & 0x7FFF) == 0x7E00 and (out[1] & 0x7FFF) == 0x7E00


# --------------------------------------------------------------------------
# the hand-derived golden blob: scales, quantiser, layout, dequantisation
# --------------------------------------------------------------------------

def _golden():
    with open(os.path.join(GOLDEN, "layout_tiny.json")) as f:
        return json.load(f)


def _golden_inputs(g):
    i = g["inputs"]
    return (np.array(i["comps"], np.float32), np.array(i["widths"], np.uint8), np.array(i["amps"], np.float32))


def test_golden_scales(orc):
    g = _golden()
    comps, widths, amps = _golden_inputs(g)
    scales, st = orc.compute_scales(comps, widths)
    assert st == 0
    assert scales.tolist() == g["scales"]


def test_golden_blob_bytes(orc):
    g = _golden()
    comps, widths, amps = _golden_inputs(g)
    scales, _ = orc.compute_scales(comps, widths)
    blob, st = orc.pack(comps, widths, scales, amps)
    assert st == 0
    expect = np.zeros(g["total_bytes"], np.uint8)
    for off, hexs in g["nonzero"].items():
        b = bytes.fromhex(hexs.replace(" ", ""))
        expect[int(off):int(off) + len(b)] = np.frombuffer(b, np.uint8)
    assert blob.size == expect.size
    diff = np.flatnonzero(blob != expect)
    assert diff.size == 0, [(int(o), int(blob[o]), int(expect[o])) for o in diff[:16]]


def test_golden_unpack_and_dequant(orc):
    g = _golden()
    comps, widths, amps = _golden_inputs(g)
    scales, _ = orc.compute_scales(comps, widths)
    blob, _ = orc.pack(comps, widths, scales, amps)
    q, w, s, a = orc.unpack(blob)
    assert q.tolist() == g["q"]
    assert w.tolist() == widths.tolist()
    for e in range(2):
        Wd, ae = orc.dequant_expert(blob, e)
        assert Wd.tolist() == g["dequant"][e]
        stored = widths[e] != 0
        assert np.array_equal(ae[stored], amps[e][stored].astype(np.float64))
        assert np.all(ae[~stored] == 0)


def test_golden_rows_layout(orc):
    """A second hand-derived blob, 40 rows and two planes: where each plane word sits."""
    with open(os.path.join(GOLDEN, "layout_rows.json")) as f:
        g = json.load(f)
    comps, widths, amps = _golden_inputs(g)
    scales, st = orc.compute_scales(comps, widths)
    assert st == 0 and scales.tolist() == g["scales"]
    blob, st = orc.pack(comps, widths, scales, amps)
    assert st == 0
    expect = np.zeros(g["total_bytes"], np.uint8)
    for off, hexs in g["nonzero"].items():
        b = bytes.fromhex(hexs.replace(" ", ""))
        expect[int(off):int(off) + len(b)] = np.frombuffer(b, np.uint8)
    assert blob.size == expect.size
    diff = np.flatnonzero(blob != expect)
    assert diff.size == 0, [(int(o), int(blob[o]), int(expect[o])) for o in diff[:16]]
    q, _, _, _ = orc.unpack(blob)
    assert q.tolist() == g["q"]


def test_golden_forward_by_hand(orc):
    """Y for one token with a hand-chosen z, worked out from the golden dequantised values."""
    g = _golden()
    comps, widths, amps = _golden_inputs(g)
    scales, _ = orc.compute_scales(comps, widths)
    blob, _ = orc.pack(comps, widths, scales, amps)
    Z = np.array([[2.0, -1.0, 0.5]])
    ids = np.array([[0, 1]], np.int32)
    gw = np.array([[0.25, 0.75]], np.float32)
    Ye, Ys, st = orc.expert_forward(blob, Z, ids, gw)
    assert st == 0
    # expert 0: 0.5*2*[0.75,-0.25,0.25] + 2.0*(-1)*[1,-2,0.5]; the 0-bit component (a=7) is absent
    y0 = np.array([0.75 - 2.0, -0.25 + 4.0, 0.25 - 1.0])
    # expert 1: 3.0*0.5*0.199951171875*[-1, 1, 1]
    y1 = 1.5 * 0.199951171875 * np.array([-1.0, 1.0, 1.0])
    assert np.array_equal(Ye[0, 0], y0)
    assert np.array_equal(Ye[0, 1], y1)
    assert np.allclose(Ys[0], 0.25 * y0 + 0.75 * y1, rtol=0, atol=1e-15)


# --------------------------------------------------------------------------
# quantiser: closed forms and brute force against "nearest mid-rise level"
# --------------------------------------------------------------------------

def test_quantiser_closed_forms(orc):
    # b=2, s=0.5: levels -0.75, -0.25, 0.25, 0.75; ties go to the upper level
    s05 = 0x3800
    cases = {0.3: 2, 0.5: 3, -0.5: 1, 0.0: 2, 0.75: 3, 10.0: 3, -10.0: 0, -0.75: 0, 0.2: 2, -0.26: 1, -0.51: 0}
    for p, q in cases.items():
        assert orc.quantise(p, 2, s05) == (q, 0), p
    # zero scale -> 0; negative / non-finite scale -> 0 with the bad-scale bit
    assert orc.quantise(0.3, 2, 0x0000) == (0, 0)
    assert orc.quantise(0.3, 2, 0x8000) == (0, 0)
    assert orc.quantise(0.3, 2, 0xB800) == (0, orc.ST_BADSCALE)
    assert orc.quantise(0.3, 2, 0x7C00) == (0, orc.ST_BADSCALE)
    assert orc.quantise(float("nan"), 2, s05) == (0, orc.ST_NONFINITE)


def test_quantiser_b1_is_sign(orc):
    rng = np.random.default_rng(7)
    for p in rng.standard_normal(200).astype(np.float32).tolist() + [0.0, -0.0]:
        q, st = orc.quantise(p, 1, 0x3C00)
        assert st == 0 and q == (1 if p >= 0 else 0)


@pytest.mark.parametrize("b", [1, 2, 3, 4, 6, 8])
def test_quantiser_is_nearest_level(orc, b):
    """Brute force over all 2^b levels in fp64: q picks the nearest level (ties up).
    Cases within 1e-5 relative of a tie are skipped: there fp32 rounding of p/s
    decides, as specified, and fp64 cannot settle it."""
    rng = np.random.default_rng(b)
    levels_q = np.arange(2 ** b)
    for _ in range(40):
        m = np.float32(abs(rng.standard_normal()) * 0.2 + 1e-3)
        s_bits = int(orc.f32_to_f16_bits(np.float32(2 * m) / np.float32(2 ** b - 1)))
        s = float(orc.f16_bits_to_f64(np.uint16(s_bits)))
        ps = (rng.uniform(-1.2, 1.2, 50) * m).astype(np.float32)
        for p in ps:
            lv = s * (levels_q - (2 ** b - 1) / 2)
            d = np.abs(float(p) - lv)
            order = np.argsort(d, kind="stable")
            if abs(d[order[0]] - d[order[1]]) <= 1e-5 * s:
                continue
            q, st = orc.quantise(float(p), b, s_bits)
            assert st == 0
            assert q == order[0], (b, float(p), s, q, order[:2])


def test_extremes_map_to_extreme_levels(orc):
    """With s = fp16(2 max|p| / (2^b-1)), the element of largest magnitude lands on
    the outermost level of its sign (closed form of the scale's definition)."""
    rng = np.random.default_rng(11)
    comps = rng.standard_normal((1, 64, 96)).astype(np.float32)
    comps /= np.linalg.norm(comps, axis=2, keepdims=True)
    for b in (1, 2, 3, 4, 6, 8):
        widths = np.full((1, 64), b, np.uint8)
        scales, st = orc.compute_scales(comps, widths)
        assert st == 0
        blob, _ = orc.pack(comps, widths, scales, np.ones((1, 64), np.float32))
        q, _, _, _ = orc.unpack(blob)
        for k in range(64):
            i = int(np.argmax(np.abs(comps[0, k])))
            expect = 2 ** b - 1 if comps[0, k, i] > 0 else 0
            assert q[0, k, i] == expect, (b, k)


def test_scale_closed_forms(orc):
    # max|p| = 0.75 at b=2 -> 0.5; max 1.5 at b=1 -> 3.0; max 0.7 at b=3 -> fp16(0.2) = 0x3266
    comps = np.zeros((1, 3, 4), np.float32)
    comps[0, 0] = [0.1, -0.75, 0.2, 0.0]
    comps[0, 1] = [1.5, -1.0, 0.0, 0.0]
    comps[0, 2] = [0.0, 0.0, -0.7, 0.1]
    widths = np.array([[2, 1, 3]], np.uint8)
    scales, st = orc.compute_scales(comps, widths)
    assert st == 0 and scales.tolist() == [[0x3800, 0x4200, 0x3266]]
    # widths 0 and 16 carry no scale; a non-finite element flags and zeroes the scale
    comps[0, 0, 0] = np.inf
    scales, st = orc.compute_scales(comps, np.array([[2, 16, 0]], np.uint8))
    assert scales.tolist() == [[0, 0, 0]] and st == orc.ST_NONFINITE


# --------------------------------------------------------------------------
# pack / unpack invariants
# --------------------------------------------------------------------------

def _random_case(rng, E, r, d_out, widths=None):
    comps = rng.standard_normal((E, r, d_out)).astype(np.float32)
    comps /= np.linalg.norm(comps, axis=2, keepdims=True)
    amps = (rng.lognormal(0, 0.5, (E, r)) * np.arange(1, r + 1) ** -0.5).astype(np.float32)
    if widths is None:
        widths = rng.choice(np.array([0, 1, 2, 3, 4, 6, 8, 16], np.uint8), size=(E, r))
    return comps, widths.astype(np.uint8), amps


@pytest.mark.parametrize("shape", [(3, 70, 13), (2, 33, 8), (1, 5, 1), (4, 100, 40)])
def test_roundtrip_and_padding(orc, shape):
    """pack -> unpack returns every q bit-exactly; no stray bit sits in padding
    (the plane popcount equals the popcount of the stored q values)."""
    rng = np.random.default_rng(sum(shape))
    E, r, d_out = shape
    comps, widths, amps = _random_case(rng, E, r, d_out)
    scales, st = orc.compute_scales(comps, widths)
    blob, st2 = orc.pack(comps, widths, scales, amps)
    assert st == 0 and st2 == 0
    q, w, s, a = orc.unpack(blob)
    assert np.array_equal(w, widths)
    qs = (widths != 0) & (widths != 16)
    assert np.array_equal(s[qs], scales[qs]) and np.all(s[~qs] == 0)
    assert np.array_equal(a[widths != 0], amps[widths != 0])
    for e in range(E):
        for k in range(r):
            b = int(widths[e, k])
            for i in range(d_out):
                if b == 0:
                    expect = 0
                elif b == 16:
                    expect = int(np.float32(comps[e, k, i]).astype(np.float16).view(np.uint16))
                else:
                    expect = orc.quantise(float(comps[e, k, i]), b, int(scales[e, k]))[0]
                assert q[e, k, i] == expect
    # padding: total set bits in all plane words == total set bits of stored q's
    n_bits_q = sum(bin(int(v)).count("1") for v in q[qs].ravel())
    n_bits_blob = _plane_popcount(blob, E)
    assert n_bits_q == n_bits_blob


def _plane_popcount(blob, E):
    """Independent reader of the format-v2 directory: popcount over every plane word."""
    blob = np.asarray(blob, np.uint8)
    d_pad = int(blob[12:16].view(np.uint32)[0])
    total = 0
    for e in range(E):
        dir_ = blob[64 + 64 * e: 128 + 64 * e]
        base = int(dir_[0:8].view(np.uint64)[0])
        goff = dir_[16:44].view(np.uint32)
        cnt = dir_[44:60].view(np.uint16)
        for gi, b in enumerate((16, 8, 6, 4, 3, 2, 1)):
            n = int(cnt[gi])
            if n == 0 or b == 16:
                continue
            npad = (n + 31) // 32 * 32
            start = base + int(goff[gi]) + 8 * npad
            words = blob[start:start + 4 * b * (npad // 32) * d_pad]
            total += int(np.unpackbits(words).sum())
    return total


def test_zero_width_contributes_exactly_zero(orc):
    """Setting the dropped components to huge values changes no byte and no output."""
    rng = np.random.default_rng(5)
    comps, widths, amps = _random_case(rng, 3, 40, 24)
    scales, _ = orc.compute_scales(comps, widths)
    blob, _ = orc.pack(comps, widths, scales, amps)
    c2, a2 = comps.copy(), amps.copy()
    c2[widths == 0] = 1e30
    a2[widths == 0] = 1e30
    s2, _ = orc.compute_scales(c2, widths)
    blob2, _ = orc.pack(c2, widths, s2, a2)
    assert np.array_equal(blob, blob2)
    Z = rng.standard_normal((2, 40))
    ids = np.array([[0, 2], [1, 0]], np.int32)
    g = np.array([[0.6, 0.4], [0.5, 0.5]], np.float32)
    Ye, Ys, _ = orc.expert_forward(blob, Z, ids, g)
    Ye2, Ys2, _ = orc.expert_forward(blob2, Z, ids, g)
    assert np.array_equal(Ye, Ye2) and np.array_equal(Ys, Ys2)


def test_blob_bytes_matches_pack_and_rejects_bad_widths(orc):
    rng = np.random.default_rng(9)
    comps, widths, amps = _random_case(rng, 2, 20, 10)
    n = orc.blob_bytes(widths, 10)
    scales, _ = orc.compute_scales(comps, widths)
    blob, _ = orc.pack(comps, widths, scales, amps)
    assert n == blob.size
    bad = widths.copy()
    bad[0, 0] = 5
    assert orc.blob_bytes(bad, 10) == 0
    with pytest.raises(orc.OracleError):
        orc.pack(comps, bad, scales, amps)


def test_blob_parse_rejects_corruption(orc):
    rng = np.random.default_rng(10)
    comps, widths, amps = _random_case(rng, 2, 20, 10)
    scales, _ = orc.compute_scales(comps, widths)
    blob, _ = orc.pack(comps, widths, scales, amps)
    for off in (0, 4, 12, 24, 64, 80, 108):
        bad = blob.copy()
        bad[off] ^= 0x5A
        with pytest.raises(orc.OracleError):
            orc.blob_dims(bad)
    with pytest.raises(orc.OracleError):
        orc.blob_dims(blob[:-16])


# --------------------------------------------------------------------------
# shared projection: closed forms and a library matmul
# --------------------------------------------------------------------------

def test_shared_proj_identity_and_one_hot(orc):
    rng = np.random.default_rng(3)
    d = 48
    eye = np.eye(d, dtype=np.float16).view(np.uint16)
    x = rng.standard_normal((3, d)).astype(np.float16)
    Z = orc.shared_proj(eye, x.view(np.uint16))
    assert np.array_equal(Z, x.astype(np.float64))  # Phi = I gives z = x exactly
    phi_t = rng.standard_normal((20, d)).astype(np.float16)
    onehot = np.zeros((1, d), np.float16)
    onehot[0, 17] = 1
    Z = orc.shared_proj(phi_t.view(np.uint16), onehot.view(np.uint16))
    assert np.array_equal(Z[0], phi_t[:, 17].astype(np.float64))


def test_shared_proj_against_numpy(orc):
    rng = np.random.default_rng(4)
    phi_t = rng.standard_normal((37, 53)).astype(np.float16)
    x = rng.standard_normal((5, 53)).astype(np.float16)
    Z = orc.shared_proj(phi_t.view(np.uint16), x.view(np.uint16))
    ref = x.astype(np.float64) @ phi_t.astype(np.float64).T
    assert np.allclose(Z, ref, rtol=1e-13, atol=1e-13)


# --------------------------------------------------------------------------
# the four checks on the factored forward
# --------------------------------------------------------------------------

def test_factored_forward_equals_dense_brute_force(orc):
    """Y_e = P_e A_e (Phi^T x) equals the dense W_e x built from the same
    dequantised factors, W_e = sum_k a_k w_k phi_k^T (first split identity)."""
    rng = np.random.default_rng(21)
    E, r, d_out, d_in, T, k = 3, 24, 16, 24, 3, 2
    comps, widths, amps = _random_case(rng, E, r, d_out)
    scales, _ = orc.compute_scales(comps, widths)
    blob, _ = orc.pack(comps, widths, scales, amps)
    phi_t = rng.standard_normal((r, d_in)).astype(np.float16)
    x = rng.standard_normal((T, d_in)).astype(np.float16)
    ids = np.array([[0, 2], [1, 1], [2, 0]], np.int32)
    g = np.array([[0.7, 0.3], [0.5, 0.5], [0.1, 0.9]], np.float32)
    Z = orc.shared_proj(phi_t.view(np.uint16), x.view(np.uint16))
    Ye, Ys, st = orc.expert_forward(blob, Z, ids, g)
    assert st == 0
    Phi = phi_t.astype(np.float64).T  # [d_in][r]
    X = x.astype(np.float64)
    for t in range(T):
        acc = np.zeros(d_out)
        for s in range(k):
            Wd, a = orc.dequant_expert(blob, int(ids[t, s]))
            W_dense = (Wd.T * a) @ Phi.T  # [d_out][d_in]
            y = W_dense @ X[t]
            assert np.allclose(Ye[t, s], y, rtol=1e-12, atol=1e-12)
            acc += float(g[t, s]) * y
        assert np.allclose(Ys[t], acc, rtol=1e-12, atol=1e-12)


def test_all_16bit_reconstructs_svd_of_stacked_experts(orc):
    """With every width at 16, the factors reconstruct each W_e of a random W_cat:
    (a) in fp64 to 1e-5 relative (the decomposition itself); (b) through fp16
    storage, packing and the oracle's forward, W_e x to 2e-3 relative."""
    rng = np.random.default_rng(31)
    E, d_out, d_in = 4, 12, 10
    W = rng.standard_normal((E, d_out, d_in))
    Phi, a, p = orc.ssd_decompose(W)
    r = Phi.shape[1]
    # (a) sum_k a_k p_k phi_k^T == W_e
    for e in range(E):
        rec = (p[e].T * a[e]) @ Phi.T
        assert np.linalg.norm(rec - W[e]) <= 1e-5 * np.linalg.norm(W[e])
    # Phi orthonormal, p unit rows (second split)
    assert np.allclose(Phi.T @ Phi, np.eye(r), atol=1e-12)
    assert np.allclose(np.linalg.norm(p, axis=2), 1.0, atol=1e-12)
    # (b) through the packed fp16 path
    widths = np.full((E, r), 16, np.uint8)
    comps = p.astype(np.float32)
    amps = a.astype(np.float32)
    scales, _ = orc.compute_scales(comps, widths)
    blob, _ = orc.pack(comps, widths, scales, amps)
    phi_t = Phi.T.astype(np.float16)
    x = rng.standard_normal((1, d_in)).astype(np.float16)
    Z = orc.shared_proj(phi_t.view(np.uint16), x.view(np.uint16))
    for e in range(E):
        _, Ys, _ = orc.expert_forward(blob, Z, np.array([[e]], np.int32), np.array([[1.0]], np.float32))
        ref = W[e] @ x[0].astype(np.float64)
        assert np.max(np.abs(Ys[0] - ref)) <= 2e-3 * np.max(np.abs(ref))


def test_single_component_closed_form(orc):
    """One stored component, one expert, g = 1: y_i = a * z * s * (q_i - (2^b-1)/2)."""
    rng = np.random.default_rng(41)
    for b in (1, 2, 3, 4, 6, 8):
        comps = rng.standard_normal((1, 1, 9)).astype(np.float32)
        widths = np.array([[b]], np.uint8)
        amps = np.array([[1.75]], np.float32)
        scales, _ = orc.compute_scales(comps, widths)
        blob, _ = orc.pack(comps, widths, scales, amps)
        q, _, _, _ = orc.unpack(blob)
        s = float(orc.f16_bits_to_f64(scales[0, 0]))
        z = 0.625
        _, Ys, _ = orc.expert_forward(blob, np.array([[z]]), np.array([[0]], np.int32),
                                      np.array([[1.0]], np.float32))
        expect = 1.75 * z * s * (q[0, 0].astype(np.float64) - (2 ** b - 1) / 2)
        assert np.array_equal(Ys[0], expect)


def test_routing_invariants(orc):
    """Permuting top-k slots permutes Y_e and keeps Y_sum; Y_sum is linear in g;
    a token alone equals the same token inside a batch; a bad id gives a zero row."""
    rng = np.random.default_rng(51)
    comps, widths, amps = _random_case(rng, 5, 30, 20)
    scales, _ = orc.compute_scales(comps, widths)
    blob, _ = orc.pack(comps, widths, scales, amps)
    Z = rng.standard_normal((3, 30))
    ids = np.array([[0, 3, 4], [2, 1, 0], [4, 4, 1]], np.int32)
    g = rng.uniform(0.1, 1, (3, 3)).astype(np.float32)
    Ye, Ys, _ = orc.expert_forward(blob, Z, ids, g)
    perm = [2, 0, 1]
    Ye2, Ys2, _ = orc.expert_forward(blob, Z, ids[:, perm], g[:, perm])
    assert np.array_equal(Ye2, Ye[:, perm])
    assert np.allclose(Ys2, Ys, rtol=1e-14, atol=1e-14)
    _, Ys3, _ = orc.expert_forward(blob, Z, ids, (2 * g).astype(np.float32))
    assert np.allclose(Ys3, 2 * Ys, rtol=1e-14, atol=1e-14)
    Ye1, Ys1, _ = orc.expert_forward(blob, Z[1:2], ids[1:2], g[1:2])
    assert np.array_equal(Ye1[0], Ye[1]) and np.array_equal(Ys1[0], Ys[1])
    bad = ids.copy()
    bad[0, 1] = 5
    Ye4, Ys4, st = orc.expert_forward(blob, Z, bad, g)
    assert st == orc.ST_BADEXPERT and np.all(Ye4[0, 1] == 0)
    assert np.allclose(Ys4[0], g[0, 0] * Ye[0, 0] + g[0, 2] * Ye[0, 2], rtol=1e-14, atol=1e-14)


def test_synth_width_counts():
    """Width counts of the workloads by cumulative rounding of their fractions."""
    from mixed_precision_decode_b200 import synth
    c = dict(synth.width_counts(synth.CONFIGS["qwen_t1"]))
    assert c == {8: 41, 4: 164, 3: 409, 2: 820, 1: 409, 0: 205}
    c = dict(synth.width_counts(synth.CONFIGS["qwen_t64"]))
    assert c == {16: 10, 8: 82, 4: 205, 3: 512, 2: 819, 1: 307, 0: 113}
    c = dict(synth.width_counts(synth.CONFIGS["mixtral_t16"]))
    assert c == {8: 205, 4: 819, 3: 1843, 2: 819, 1: 410}
    c = dict(synth.width_counts(synth.CONFIGS["tiny"]))
    assert c == {b: 8 for b in (16, 8, 6, 4, 3, 2, 1, 0)}


def test_synth_tiny_layer_shapes():
    from mixed_precision_decode_b200 import synth
    L = synth.make_layer(synth.CONFIGS["tiny"])
    assert L["gate"]["phi_t"].shape == (64, 64) and L["gate"]["comps"].shape == (4, 64, 32)
    w = L["gate"]["widths"]
    for e in range(4):
        vals, cnt = np.unique(w[e].numpy(), return_counts=True)
        assert dict(zip(vals.tolist(), cnt.tolist())) == {b: 8 for b in (0, 1, 2, 3, 4, 6, 8, 16)}
        order = np.argsort(-L["gate"]["amps"][e].numpy(), kind="stable")
        assert w[e].numpy()[order[:8]].tolist() == [16] * 8
    assert L["ids"].shape == (4, 2) and np.allclose(L["gate_w"].sum(1).numpy(), 1, atol=1e-6)


# --------------------------------------------------------------------------
# expert FFN output: SiLU(gate) * up, then the dense down projection
# --------------------------------------------------------------------------

def test_ffn_silu_closed_forms(orc):
    """With an identity down matrix and g = 1 the output is SiLU(y_g) * y_u per
    column.  The logistic function has closed forms at ln 3 (3/4), -ln 3 (1/4)
    and 0 (1/2); far out it saturates to 1 (v = 40: v exactly) and to 0 without
    an overflow NaN (v = -800).  Gate and up enter asymmetrically, so swapping
    them fails the first column."""
    ln3 = np.log(3.0)
    W = np.eye(6, dtype=np.float16).view(np.uint16)[None]
    Yg = np.array([[[ln3, -ln3, 0.0, 40.0, -800.0, 1.0]]])
    Yu = np.array([[[1.0, 2.0, -3.0, 0.5, 7.0, ln3]]])
    out, st = orc.ffn_down(Yg, Yu, W, np.zeros((1, 1), np.int32), np.ones((1, 1), np.float32))
    assert st == 0
    expect = np.array([0.75 * ln3, -0.5 * ln3, 0.0, 20.0, 0.0, ln3 / (1 + np.exp(-1.0))])
    assert np.allclose(out[0, :4], expect[:4], rtol=1e-15, atol=0)
    assert out[0, 4] == 0.0 and np.isfinite(out).all()
    assert abs(out[0, 5] - expect[5]) <= 1e-15 * abs(expect[5])


def _dense_gate_up(orc, blob, e, Phi):
    Wd, a = orc.dequant_expert(blob, e)
    return (Wd.T * a) @ Phi.T  # [d_out][d_in]


def test_ffn_matches_dense_expert_brute_force(orc):
    """The oracle's whole expert FFN (spectral gate/up, then SiLU(gate) * up and the
    down projection) equals the textbook dense gated expert built from the same
    dequantised factors: out = sum_s g_s Wd_e (silu(Wg_e x) * (Wu_e x)), with
    SiLU from scipy's logistic function and numpy matmuls, on a non-square case
    (d_model = 24 != d_ff = 16) so a transposed operand cannot pass."""
    from scipy.special import expit
    rng = np.random.default_rng(61)
    E, r, d_ff, d_model, T = 3, 24, 16, 24, 3
    blobs = {}
    for name in ("gate", "up"):
        comps, widths, amps = _random_case(rng, E, r, d_ff)
        scales, _ = orc.compute_scales(comps, widths)
        blobs[name], _ = orc.pack(comps, widths, scales, amps)
    phi_t = {n: rng.standard_normal((r, d_model)).astype(np.float16) for n in ("gate", "up")}
    w_down = (rng.standard_normal((E, d_model, d_ff)) / 4).astype(np.float16)
    x = rng.standard_normal((T, d_model)).astype(np.float16)
    ids = np.array([[0, 2], [1, 1], [2, 0]], np.int32)
    g = np.array([[0.7, 0.3], [0.5, 0.5], [0.1, 0.9]], np.float32)
    out, st = orc.moe_ffn_forward(blobs["gate"], blobs["up"], phi_t["gate"].view(np.uint16),
                                  phi_t["up"].view(np.uint16), x.view(np.uint16), ids, g, w_down.view(np.uint16))
    assert st == 0 and out.shape == (T, d_model)
    X = x.astype(np.float64)
    for t in range(T):
        ref = np.zeros(d_model)
        for s in range(ids.shape[1]):
            e = int(ids[t, s])
            yg = _dense_gate_up(orc, blobs["gate"], e, phi_t["gate"].astype(np.float64).T) @ X[t]
            yu = _dense_gate_up(orc, blobs["up"], e, phi_t["up"].astype(np.float64).T) @ X[t]
            h = yg * expit(yg) * yu
            ref += float(g[t, s]) * (w_down[e].astype(np.float64) @ h)
        assert np.max(np.abs(out[t] - ref)) <= 1e-12 * np.max(np.abs(ref))


def test_ffn_routing_invariants(orc):
    """Permuting the top-k slots keeps the output; it is linear in g and in the
    down matrix; a token alone equals the same token in a batch; an id out of
    range drops its slot and sets the status bit; T = 0 gives an empty output."""
    rng = np.random.default_rng(71)
    E, d_model, d_ff, T, K = 4, 10, 12, 3, 3
    W = (rng.standard_normal((E, d_model, d_ff)) / 3).astype(np.float16)
    Yg = rng.standard_normal((T, K, d_ff)) * 2
    Yu = rng.standard_normal((T, K, d_ff))
    ids = np.array([[0, 3, 1], [2, 2, 0], [3, 1, 0]], np.int32)
    g = rng.uniform(0.1, 1, (T, K)).astype(np.float32)
    out, st = orc.ffn_down(Yg, Yu, W.view(np.uint16), ids, g)
    assert st == 0
    perm = [2, 0, 1]
    out2, _ = orc.ffn_down(Yg[:, perm], Yu[:, perm], W.view(np.uint16), ids[:, perm], g[:, perm])
    assert np.allclose(out2, out, rtol=1e-14, atol=1e-14)
    out3, _ = orc.ffn_down(Yg, Yu, W.view(np.uint16), ids, (2 * g).astype(np.float32))
    assert np.allclose(out3, 2 * out, rtol=1e-14, atol=1e-14)
    W2 = (2 * W.astype(np.float32)).astype(np.float16)  # exact: a power-of-two scaling
    out4, _ = orc.ffn_down(Yg, Yu, W2.view(np.uint16), ids, g)
    assert np.array_equal(out4, 2 * out)
    out1, _ = orc.ffn_down(Yg[1:2], Yu[1:2], W.view(np.uint16), ids[1:2], g[1:2])
    assert np.array_equal(out1[0], out[1])
    bad = ids.copy()
    bad[0, 1] = E
    out5, st5 = orc.ffn_down(Yg, Yu, W.view(np.uint16), bad, g)
    assert st5 == orc.ST_BADEXPERT
    keep = [0, 2]
    out6, _ = orc.ffn_down(Yg[:1, keep], Yu[:1, keep], W.view(np.uint16), ids[:1, keep], g[:1, keep])
    assert np.allclose(out5[0], out6[0], rtol=1e-14, atol=1e-14) and np.array_equal(out5[1:], out[1:])
    out0, st0 = orc.ffn_down(Yg[:0], Yu[:0], W.view(np.uint16), ids[:0], g[:0])
    assert out0.shape == (0, d_model) and st0 == 0


# --------------------------------------------------------------------------
# widths by descending amplitude (the configurations' allocation rule)
# --------------------------------------------------------------------------

def test_assign_widths_brute_force(orc):
    """Per expert: the counts per width are exact; a component never gets a width
    listed later than one of smaller amplitude; among equal amplitudes the lower k
    comes first.  Checked against every pair of components."""
    rng = np.random.default_rng(81)
    order, counts = (8, 4, 3, 2, 1, 0), (1, 2, 3, 4, 2, 2)
    a = rng.choice([0.5, 1.0, 1.5, 2.0, 3.0], size=(3, 14)).astype(np.float32)  # many ties
    w = orc.assign_widths(a, order, counts)
    rank = {b: i for i, b in enumerate(order)}
    for e in range(3):
        assert [int((w[e] == b).sum()) for b in order] == list(counts)
        for j in range(14):
            for k in range(14):
                if a[e, j] > a[e, k] or (a[e, j] == a[e, k] and j < k):
                    assert rank[int(w[e, j])] <= rank[int(w[e, k])]


# --------------------------------------------------------------------------
# FQCM: distortion per width, activation importance, the bit-budget allocation
# --------------------------------------------------------------------------

def test_fqcm_eps_closed_forms(orc):
    """p = (1.5, -1.5, 0.5, -0.5): at 2 bits the scale is fp16(3 / 3) = 1 and the levels
    are +-0.5, +-1.5, so eps = 0; at 1 bit the levels are +-1.5 (scale 3) and the two
    small entries land on the far levels, eps = 1 + 1 = 2; at 0 bits eps = ||p||^2 = 5;
    every entry is an fp16 value, so eps(16) = 0.  p = (1.5, 0.2, 0, 0) at 2 bits: 0.2 and
    both zeros go to level 0.5 (the mid-rise levels have no 0), eps = 0.3^2 + 2 (0.5)^2.
    fp16 rounding of 0.1 against numpy's float16."""
    p = np.zeros((1, 3, 4), np.float32)
    p[0, 0] = [1.5, -1.5, 0.5, -0.5]
    p[0, 1] = [1.5, 0.2, 0.0, 0.0]
    p[0, 2] = [0.1, 0.0, 0.0, 0.0]
    eps = orc.fqcm_eps(p)
    W = {b: i for i, b in enumerate(orc.WIDTH_SET)}
    assert eps[0, 0, W[2]] == 0.0 and eps[0, 0, W[16]] == 0.0
    assert eps[0, 0, W[1]] == 2.0 and eps[0, 0, W[0]] == 5.0
    assert abs(eps[0, 1, W[2]] - ((float(np.float32(0.2)) - 0.5) ** 2 + 2 * 0.25)) <= 1e-15
    h = float(np.float16(np.float32(0.1)))
    assert eps[0, 2, W[16]] == (float(np.float32(0.1)) - h) ** 2


def test_fqcm_eps_falls_with_width_on_average(orc):
    """On random unit vectors eps falls with every width from 2 bits on.  At 1 bit the
    mid-rise levels are +-max|p|, which overshoot most entries: on average eps(1) is
    above eps(0) = ||p||^2 = 1 (so an allocation never prefers 1 bit to 0 there)."""
    rng = np.random.default_rng(91)
    p = rng.standard_normal((2, 50, 64)).astype(np.float32)
    p /= np.linalg.norm(p, axis=2, keepdims=True)
    m = orc.fqcm_eps(p).mean(axis=(0, 1))
    assert abs(m[0] - 1.0) <= 1e-6 and m[1] > m[0] and np.all(np.diff(m[1:]) < 0)


def test_fqcm_beta_closed_form_and_H_route(orc):
    """beta[e][k] = sum over pairs routed to e of g z_k^2 (a closed form on a 2 x 2 case),
    and equal to diag(Phi^T H_e Phi) with H_e = sum g x x^T built by numpy matmuls."""
    Z = np.array([[1.0, 2.0], [3.0, 0.0]])
    ids = np.array([[0, 1], [1, 0]])
    g = np.array([[0.5, 0.25], [1.0, 2.0]])
    beta = orc.fqcm_beta(Z, ids, g, 2)
    assert np.array_equal(beta, np.array([[18.5, 2.0], [9.25, 1.0]]))
    rng = np.random.default_rng(92)
    T, d_in, r, E, K = 6, 10, 7, 3, 2
    X = rng.standard_normal((T, d_in))
    Phi, _ = np.linalg.qr(rng.standard_normal((d_in, r)))
    ids = rng.integers(0, E, (T, K))
    g = rng.uniform(0, 1, (T, K))
    beta = orc.fqcm_beta(X @ Phi, ids, g, E)
    for e in range(E):
        H = sum(g[t, j] * np.outer(X[t], X[t]) for t in range(T) for j in range(K) if ids[t, j] == e)
        H = H if not np.isscalar(H) else np.zeros((d_in, d_in))
        assert np.allclose(beta[e], np.diag(Phi.T @ H @ Phi), rtol=1e-12, atol=1e-12)


def _brute(a, beta, eps, d_out, budget, WS):
    import itertools
    E, r = a.shape
    best = None
    for combo in itertools.product(range(8), repeat=E * r):
        bits = sum(d_out * WS[i] for i in combo)
        if bits > budget:
            continue
        loss = sum(a[c // r, c % r] ** 2 * beta[c // r, c % r] * eps[c // r, c % r, i] for c, i in enumerate(combo))
        best = loss if best is None else min(best, loss)
    return best


def test_allocate_widths_optimal_at_relaxation_vertices(orc):
    """Brute force over all 8^4 width choices: at every budget where the relaxation's
    solution is integral (the cumulative bits of its first m steps) the allocation is
    optimal; at any budget it respects the budget and more budget never costs loss."""
    rng = np.random.default_rng(93)
    WS = orc.WIDTH_SET
    E, r, d_out = 1, 4, 2
    a = rng.uniform(0.2, 2.0, (E, r))
    beta = rng.uniform(0.1, 3.0, (E, r))
    eps = np.sort(rng.uniform(0, 1, (E, r, 8)), axis=2)[:, :, ::-1].copy()  # falling with width
    eps[:, :, 0] = 1.0
    prev = None
    vertices = 0
    for budget in range(0, d_out * 16 * r + 1, 2):
        w, loss = orc.allocate_widths(a, beta, eps, d_out, budget)
        used = int(d_out * w.astype(np.int64).sum())
        assert used <= budget
        if prev is not None:
            assert loss <= prev + 1e-12
        prev = loss
        if used == budget:  # the relaxation's solution is integral here
            vertices += 1
            assert abs(loss - _brute(a, beta, eps, d_out, budget, WS)) <= 1e-12
    assert vertices >= 8


def test_allocate_widths_edges(orc):
    E, r, d_out = 2, 3, 4
    a = np.ones((E, r))
    eps = np.tile(np.linspace(1, 0, 8), (E, r, 1))
    w, loss = orc.allocate_widths(a, np.zeros((E, r)), eps, d_out, 10 ** 6)
    assert np.all(w == 0) and loss == 0.0  # no importance: nothing is worth a bit
    w, _ = orc.allocate_widths(a, np.ones((E, r)), eps, d_out, 0)
    assert np.all(w == 0)
    w, loss = orc.allocate_widths(a, np.ones((E, r)), eps, d_out, 10 ** 6)
    assert np.all(w == 16) and loss == 0.0
