"""The C ABI on the host (no GPU): the library builds, loads and exports every
symbol include/bitsmoe.h declares; plans and argument checks behave as the
header says; the plan's header+directory equals the oracle's byte for byte."""
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def B():
    from mixed_precision_decode_b200 import build
    build.build()
    from mixed_precision_decode_b200 import bitsmoe
    return bitsmoe


def _declared():
    src = open(os.path.join(ROOT, "include", "bitsmoe.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(bitsmoe_[a-z_0-9]+)\s*\(", src)))


def test_exports_every_declared_symbol(B):
    import ctypes
    L = ctypes.CDLL(B._LIB_PATH)
    declared = _declared()
    assert len(declared) >= 18
    for name in declared:
        assert hasattr(L, name), name
    assert sorted(B.EXPORTS) == declared
    assert B.version() == 100


def test_checked_build_exports_the_same_symbols(B):
    """The bounds-checked library is the same C ABI (only the kernels differ)."""
    import ctypes
    from mixed_precision_decode_b200 import build
    path = build.build(checked=True)
    L = ctypes.CDLL(path)
    for name in _declared():
        assert hasattr(L, name), name
    L.bitsmoe_version.restype = ctypes.c_int
    assert L.bitsmoe_version() == 100


def _widths(rng, E, r):
    return rng.choice(np.array([0, 1, 2, 3, 4, 6, 8, 16], np.uint8), size=(E, r))


@pytest.mark.parametrize("shape", [(1, 1, 1), (3, 70, 13), (5, 100, 40), (2, 64, 32)])
def test_plan_header_matches_oracle(B, orc, shape):
    E, r, d_out = shape
    rng = np.random.default_rng(E * 1000 + r)
    w = _widths(rng, E, r)
    comps = rng.standard_normal((E, r, d_out)).astype(np.float32)
    amps = np.ones((E, r), np.float32)
    scales, _ = orc.compute_scales(comps, w)
    blob, _ = orc.pack(comps, w, scales, amps)
    plan = B.pack_plan(8, d_out, E, r, 2, w)
    assert plan.blob_bytes == blob.size == orc.blob_bytes(w, d_out)
    assert plan.header_bytes == 64 + 64 * E
    assert np.array_equal(plan.header(), blob[:64 + 64 * E])
    d = plan.dims
    assert (d.d_in, d.d_out, d.n_experts, d.rank, d.top_k) == (8, d_out, E, r, 2)
    # a saved blob's header rebuilds the same plan
    p2 = B.plan_from_header(blob[:plan.header_bytes], 8, 2)
    assert p2.blob_bytes == plan.blob_bytes and np.array_equal(p2.header(), plan.header())


def test_plan_errors(B):
    w = np.zeros((2, 4), np.uint8)
    with pytest.raises(B.BitsMoEError) as ei:
        B.pack_plan(8, 4, 2, 4, 1, np.full((2, 4), 5, np.uint8))
    assert ei.value.code == B.EWIDTH
    for bad in [(0, 4, 2, 4, 1), (8, 0, 2, 4, 1), (8, 4, 0, 4, 1), (8, 4, 2, 0, 1), (8, 4, 2, 4, 0),
                (8, 4, 2, 70000, 1)]:
        with pytest.raises(B.BitsMoEError) as ei:
            B.pack_plan(*bad, np.zeros((max(bad[2], 1), max(min(bad[3], 70000), 1)), np.uint8))
        assert ei.value.code == B.EINVAL
    plan = B.pack_plan(8, 4, 2, 4, 1, w)
    hdr = plan.header()
    bad = hdr.copy()
    bad[0] ^= 1
    with pytest.raises(B.BitsMoEError) as ei:
        B.plan_from_header(bad, 8, 1)
    assert ei.value.code == B.EFORMAT
    bad = hdr.copy()
    bad[64 + 44] += 1  # a count that no longer sums to r
    with pytest.raises(B.BitsMoEError) as ei:
        B.plan_from_header(bad, 8, 1)
    assert ei.value.code == B.EFORMAT
    with pytest.raises(B.BitsMoEError) as ei:
        B.plan_from_header(hdr[:100], 8, 1)
    assert ei.value.code == B.ESIZE


def test_argument_checks_before_any_launch(B):
    """NULL and misaligned pointers and bad dims are refused on the host."""
    import ctypes
    L = B.lib()
    w = np.zeros((2, 4), np.uint8)
    w[:, :2] = 2
    plan = B.pack_plan(8, 4, 2, 4, 1, w)
    h = plan.handle
    assert L.bitsmoe_pack(h, None, None, None, None, None, None, None) == B.EINVAL
    assert L.bitsmoe_pack(h, 16, 16, 16, 16, 0x1001, None, None) == B.EINVAL  # blob not 16-byte aligned
    assert L.bitsmoe_compute_scales(None, 16, 16, 16, None, None) == B.EINVAL
    assert L.bitsmoe_unpack_q(h, None, 16, None) == B.EINVAL
    assert L.bitsmoe_shared_proj(16, 16, 16, -1, 8, 4, None) == B.EINVAL
    assert L.bitsmoe_shared_proj(16, 16, 16, 1, 12, 4, None) == B.EINVAL  # d_in % 8
    assert L.bitsmoe_shared_proj(0x1008, 16, 16, 1, 8, 4, None) == B.EINVAL  # phi_t misaligned
    assert L.bitsmoe_shared_proj(None, None, None, 0, 8, 4, None) == B.OK  # T = 0: no-op
    need = B.expert_workspace_bytes(plan, 3)
    assert need > 0
    assert L.bitsmoe_expert_forward(h, 256, 256, 256, 256, 3, None, 256, 256, need - 1, None, None) == B.ESIZE
    assert L.bitsmoe_expert_forward(h, 256, 256, 256, 256, 3, None, 256, 0x1010, need, None, None) == B.EINVAL
    assert L.bitsmoe_expert_forward(h, 256, 256, 256, 256, 0, None, 256, None, 0, None, None) == B.OK
    assert L.bitsmoe_read_status(None, None, ctypes.byref(ctypes.c_int32())) == B.EINVAL
    io = B.proj_io(plan, 256, 256, 256)
    io_bad = B.proj_io(plan, 0x1008, 256, 256)
    assert L.bitsmoe_layer_forward(ctypes.byref(io), ctypes.byref(io_bad), 256, 256, 256, 1, 256, 1 << 20, None,
                                   None) == B.EINVAL
    nl = B.layer_workspace_bytes(plan, plan, 2)
    assert L.bitsmoe_layer_forward(ctypes.byref(io), ctypes.byref(io), 256, 256, 256, 2, 256, nl - 1, None,
                                   None) == B.ESIZE
    assert B.strerror(B.EWIDTH).startswith("width")


def test_chained_call_rejects_one_next_pointer(B):
    """The next-layer pointers come in pairs and are 16-byte aligned; the checks run
    before any device work."""
    L = B.lib()
    rc = L.bitsmoe_layer_forward_chained(None, None, None, None, None, 1, None, 0, 256, None, None, None)
    assert rc == B.EINVAL
    rc = L.bitsmoe_layer_forward_chained(None, None, None, None, None, 1, None, 0, 256, 264, None, None)
    assert rc == B.EINVAL


def test_workspace_holds_the_multi_token_c_rows(B):
    """The expert and layer workspaces hold, per routed pair, a c row as long as the
    largest expert's padded member list (rounded up to 8 floats), its zero-point
    total and its output row."""
    rng = np.random.default_rng(7)
    E, r, d_out, K = 5, 100, 40, 2
    w = _widths(rng, E, r)
    plan = B.pack_plan(8, d_out, E, r, K, w)

    def padded(b, n):
        return 0 if n == 0 else (-(-n // 8) * 8 if b == 16 else -(-n // 32) * 32)

    members = max(sum(padded(int(b), int((w[e] == b).sum())) for b in (16, 8, 6, 4, 3, 2, 1)) for e in range(E))
    ldc = -(-members // 8) * 8
    for T in (1, 3, 17):
        per_pair = 4 * ldc + 4 + 4 * d_out
        assert B.expert_workspace_bytes(plan, T) >= T * K * per_pair
        assert B.layer_workspace_bytes(plan, plan, T) >= T * K * (4 * ldc + 4)
    # each buffer is rounded up to 256 bytes: the growth may fall short by that per buffer
    grow = B.expert_workspace_bytes(plan, 17) - B.expert_workspace_bytes(plan, 3)
    assert grow >= 14 * K * per_pair - 3 * 256


def test_ffn_down_argument_checks_and_sizes(B):
    """The down step's dims, pointer and workspace checks run on the host before any
    launch; launch counts and workspace sizes follow the two paths."""
    import ctypes
    L = B.lib()
    q = B.ffn_dims(2048, 768, 128, 8)
    assert B.ffn_down_launches(q, 0) == 0 and B.ffn_down_launches(q, 1) == 1 and B.ffn_down_launches(q, 64) == 3
    assert B.ffn_down_workspace_bytes(q, 1) == 0
    n64 = B.ffn_down_workspace_bytes(q, 64)
    assert n64 >= 64 * 8 * 2048 * 4 + 64 * 8 * 4  # per-pair down rows and the pair lists
    big = B.ffn_dims(96, 8192, 8, 8)  # top_k x d_ff beyond one CTA: grouped kernels even at T = 1
    assert B.ffn_down_launches(big, 1) == 3 and B.ffn_down_workspace_bytes(big, 1) > 0
    bad = B.ffn_dims(64, 12, 4, 2)  # d_ff % 8
    assert L.bitsmoe_ffn_down_launches(ctypes.byref(bad), 1) == B.EINVAL
    assert L.bitsmoe_ffn_down(ctypes.byref(bad), 256, 256, 256, 256, 256, 1, 256, None, 0, None, None) == B.EINVAL
    assert L.bitsmoe_ffn_down(ctypes.byref(q), None, None, None, None, None, 0, None, None, 0, None, None) == B.OK
    assert L.bitsmoe_ffn_down(ctypes.byref(q), None, 256, 256, 256, 256, 1, 256, None, 0, None, None) == B.EINVAL
    assert L.bitsmoe_ffn_down(ctypes.byref(q), 256, 0x1004, 256, 256, 256, 1, 256, None, 0, None,
                              None) == B.EINVAL  # Y_gate misaligned
    assert L.bitsmoe_ffn_down(ctypes.byref(q), 256, 256, 256, 256, 256, 64, 256, 512, n64 - 1, None,
                              None) == B.ESIZE
    assert L.bitsmoe_ffn_down(ctypes.byref(q), 256, 256, 256, 256, 256, 64, 256, 0x1010, n64, None,
                              None) == B.EINVAL  # workspace not 256-byte aligned
    assert L.bitsmoe_ffn_down(ctypes.byref(q), 256, 256, 256, 256, 256, -1, 256, None, 0, None, None) == B.EINVAL


def test_ffn_forward_argument_checks(B):
    """The whole-FFN call needs both projections' per-slot outputs and an aligned
    down matrix; T = 0 is a no-op; the workspace is the layer's plus the down step's."""
    import ctypes
    L = B.lib()
    w = np.zeros((2, 8), np.uint8)
    w[:, :4] = 2
    plan = B.pack_plan(16, 8, 2, 8, 1, w)
    nl, nf = B.layer_workspace_bytes(plan, plan, 3), B.ffn_workspace_bytes(plan, plan, 3)
    assert nf >= nl + 3 * 1 * 16 * 4
    assert B.ffn_launches(plan, plan, 1) == B.layer_launches(plan, plan, 1) + 1
    assert B.ffn_launches(plan, plan, 3) == B.layer_launches(plan, plan, 3) + 3
    io = B.proj_io(plan, 256, 256, 256, Y_experts=256)
    io_noy = B.proj_io(plan, 256, 256, 256)
    args = (256, 256, 256, 256, 3, 256, 512, nf, None, None)
    assert L.bitsmoe_ffn_forward(ctypes.byref(io), ctypes.byref(io), 256, 256, 256, 256, 0, 256, None, 0, None,
                                 None) == B.OK
    assert L.bitsmoe_ffn_forward(ctypes.byref(io), ctypes.byref(io_noy), *args) == B.EINVAL
    assert L.bitsmoe_ffn_forward(ctypes.byref(io), ctypes.byref(io), 0x1008, 256, 256, 256, 3, 256, 512, nf, None,
                                 None) == B.EINVAL  # w_down misaligned
    assert L.bitsmoe_ffn_forward(ctypes.byref(io), ctypes.byref(io), 256, 256, 256, 256, 3, 256, 512, nf - 1, None,
                                 None) == B.ESIZE
