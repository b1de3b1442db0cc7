"""Oracle: a plain, slow CPU reference of the BitsMoE spectral MoE gate/up decode path.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The product library
(``mixed_precision_decode_b200``) never imports, loads or calls it, and the two
share no code: the bit-level work (fp16 conversion, scales, quantiser, packing,
unpacking, the fp64 forward) is in ``bitsmoe_oracle.c``, compiled here with gcc;
the offline shared-basis decomposition used by the reconstruction check is
below, written with numpy's SVD as its one library primitive.

Method sources (the BitsMoE study-note page, "BitsMoE: Cost-Aware Bit
Allocation In spectral Space for MoE LLM Quantization"):

* Methodology, first split -- stack the E expert matrices of one projection
  into W_cat, take its SVD W_cat = U S Phi^T; with P = U S, W_e x = P_e (Phi^T x).
* second split -- normalise each column of P_e: W_e = sum_k a_{e,k} p_{e,k} phi_k^T,
  ||p_{e,k}|| = 1.
* Usage -- widths {0,1,2,3,4,6,8,16}: 0 drops the component, 16 keeps fp16.
* Execution -- equal widths grouped, packed by bit plane.

Every function here is pinned by ``tests/test_oracle.py``; none is "parity
unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "bitsmoe_oracle.c")
_LIB = os.path.join(_HERE, "libbitsmoe_oracle.so")

# Status bits and error codes, as the oracle's C file defines them.
ST_NONFINITE = 1
ST_BADSCALE = 2
ST_BADEXPERT = 4

WIDTHS = (0, 1, 2, 3, 4, 6, 8, 16)
GROUP_ORDER = (16, 8, 6, 4, 3, 2, 1)


def build(force: bool = False) -> str:
    """Compile the oracle's C file into a shared library next to it."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
             "-Wall", "-Wextra", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        c_u8p = ctypes.POINTER(ctypes.c_uint8)
        c_u16p = ctypes.POINTER(ctypes.c_uint16)
        c_i32p = ctypes.POINTER(ctypes.c_int32)
        c_f32p = ctypes.POINTER(ctypes.c_float)
        c_f64p = ctypes.POINTER(ctypes.c_double)
        L.orc_f32_to_f16.argtypes = [ctypes.c_float]
        L.orc_f32_to_f16.restype = ctypes.c_uint16
        L.orc_f16_to_f64.argtypes = [ctypes.c_uint16]
        L.orc_f16_to_f64.restype = ctypes.c_double
        L.orc_quantise.argtypes = [ctypes.c_float, ctypes.c_int, ctypes.c_uint16, c_i32p]
        L.orc_quantise.restype = ctypes.c_uint32
        L.orc_blob_bytes.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, c_u8p]
        L.orc_blob_bytes.restype = ctypes.c_uint64
        L.orc_compute_scales.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, c_f32p, c_u8p, c_u16p, c_i32p]
        L.orc_pack.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, c_u8p, c_f32p, c_u16p, c_f32p, c_u8p,
                               ctypes.c_uint64, c_i32p]
        L.orc_blob_parse.argtypes = [c_u8p, ctypes.c_uint64, c_i32p, c_i32p, c_i32p]
        L.orc_unpack.argtypes = [c_u8p, ctypes.c_uint64, c_u16p, c_u8p, c_u16p, c_f32p]
        L.orc_dequant_expert.argtypes = [c_u8p, ctypes.c_uint64, ctypes.c_int, c_f64p, c_f64p]
        L.orc_shared_proj.argtypes = [c_u16p, c_u16p, ctypes.c_int, ctypes.c_int, ctypes.c_int, c_f64p]
        L.orc_shared_proj.restype = None
        L.orc_expert_forward.argtypes = [c_u8p, ctypes.c_uint64, c_f64p, c_i32p, c_f32p, ctypes.c_int,
                                         ctypes.c_int, c_f64p, c_f64p, c_i32p]
        L.orc_fqcm_eps.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, c_f32p, c_f64p]
        L.orc_ffn_down.argtypes = [c_f64p, c_f64p, c_u16p, c_i32p, c_f32p, ctypes.c_int, ctypes.c_int,
                                   ctypes.c_int, ctypes.c_int, ctypes.c_int, c_f64p, c_i32p]
        for f in ("orc_compute_scales", "orc_pack", "orc_blob_parse", "orc_unpack", "orc_dequant_expert",
                  "orc_expert_forward", "orc_ffn_down", "orc_fqcm_eps"):
            getattr(L, f).restype = ctypes.c_int
        _lib = L
    return _lib


def _p(a: np.ndarray, ct):
    return a.ctypes.data_as(ctypes.POINTER(ct))


def _c(a, dtype) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=dtype)


class OracleError(RuntimeError):
    pass


def _check(rc: int, what: str):
    if rc != 0:
        raise OracleError(f"{what} failed with code {rc}")


# ---------------------------------------------------------------------------
# fp16
# ---------------------------------------------------------------------------

def f32_to_f16_bits(x) -> np.ndarray:
    """fp32 -> fp16 bits, round to nearest even (the oracle's own converter)."""
    x = np.asarray(x, dtype=np.float32)
    f = lib().orc_f32_to_f16
    out = np.fromiter((f(float(v)) for v in x.ravel()), dtype=np.uint16, count=x.size)
    return out.reshape(x.shape)


def f16_bits_to_f64(h) -> np.ndarray:
    h = np.asarray(h, dtype=np.uint16)
    f = lib().orc_f16_to_f64
    out = np.fromiter((f(int(v)) for v in h.ravel()), dtype=np.float64, count=h.size)
    return out.reshape(h.shape)


def quantise(p: float, b: int, scale_bits: int) -> tuple[int, int]:
    """Quantise one element; returns (q, status bits)."""
    st = ctypes.c_int32(0)
    q = lib().orc_quantise(ctypes.c_float(p), b, scale_bits, ctypes.byref(st))
    return int(q), int(st.value)


# ---------------------------------------------------------------------------
# scales, pack, unpack
# ---------------------------------------------------------------------------

def blob_bytes(widths: np.ndarray, d_out: int) -> int:
    w = _c(widths, np.uint8)
    E, r = w.shape
    return int(lib().orc_blob_bytes(E, r, d_out, _p(w, ctypes.c_uint8)))


def compute_scales(comps: np.ndarray, widths: np.ndarray) -> tuple[np.ndarray, int]:
    """fp16 scale bits [E][r] from comps [E][r][d_out] (fp32); returns (scales, status)."""
    comps = _c(comps, np.float32)
    w = _c(widths, np.uint8)
    E, r, d_out = comps.shape
    scales = np.zeros((E, r), np.uint16)
    st = ctypes.c_int32(0)
    _check(lib().orc_compute_scales(E, r, d_out, _p(comps, ctypes.c_float), _p(w, ctypes.c_uint8),
                                    _p(scales, ctypes.c_uint16), ctypes.byref(st)), "compute_scales")
    return scales, int(st.value)


def pack(comps: np.ndarray, widths: np.ndarray, scales: np.ndarray, amps: np.ndarray) -> tuple[np.ndarray, int]:
    """Pack into the format-v2 blob; returns (blob uint8, status)."""
    comps = _c(comps, np.float32)
    w = _c(widths, np.uint8)
    s = _c(scales, np.uint16)
    a = _c(amps, np.float32)
    E, r, d_out = comps.shape
    n = blob_bytes(w, d_out)
    if n == 0:
        raise OracleError("invalid widths or dims")
    blob = np.zeros(n, np.uint8)
    st = ctypes.c_int32(0)
    _check(lib().orc_pack(E, r, d_out, _p(w, ctypes.c_uint8), _p(comps, ctypes.c_float), _p(s, ctypes.c_uint16),
                          _p(a, ctypes.c_float), _p(blob, ctypes.c_uint8), n, ctypes.byref(st)), "pack")
    return blob, int(st.value)


def blob_dims(blob: np.ndarray) -> tuple[int, int, int]:
    blob = _c(blob, np.uint8)
    E, r, d = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int32()
    _check(lib().orc_blob_parse(_p(blob, ctypes.c_uint8), blob.size, ctypes.byref(E), ctypes.byref(r),
                                ctypes.byref(d)), "blob_parse")
    return E.value, r.value, d.value


def unpack(blob: np.ndarray):
    """Returns (q [E][r][d_out] u16, widths [E][r], scales [E][r], amps [E][r])."""
    blob = _c(blob, np.uint8)
    E, r, d_out = blob_dims(blob)
    q = np.zeros((E, r, d_out), np.uint16)
    w = np.zeros((E, r), np.uint8)
    s = np.zeros((E, r), np.uint16)
    a = np.zeros((E, r), np.float32)
    _check(lib().orc_unpack(_p(blob, ctypes.c_uint8), blob.size, _p(q, ctypes.c_uint16), _p(w, ctypes.c_uint8),
                            _p(s, ctypes.c_uint16), _p(a, ctypes.c_float)), "unpack")
    return q, w, s, a


def dequant_expert(blob: np.ndarray, e: int) -> tuple[np.ndarray, np.ndarray]:
    """Dequantised directions Wd [r][d_out] (fp64) and amplitudes a [r] of expert e."""
    blob = _c(blob, np.uint8)
    E, r, d_out = blob_dims(blob)
    Wd = np.zeros((r, d_out), np.float64)
    a = np.zeros(r, np.float64)
    _check(lib().orc_dequant_expert(_p(blob, ctypes.c_uint8), blob.size, e, _p(Wd, ctypes.c_double),
                                    _p(a, ctypes.c_double)), "dequant_expert")
    return Wd, a


# ---------------------------------------------------------------------------
# forward
# ---------------------------------------------------------------------------

def shared_proj(phi_t_bits: np.ndarray, x_bits: np.ndarray) -> np.ndarray:
    """Z [T][r] (fp64) = Phi^T x per token; phi_t [r][d_in], x [T][d_in] fp16 bits."""
    P = _c(phi_t_bits, np.uint16)
    X = _c(x_bits, np.uint16)
    r, d_in = P.shape
    T = X.shape[0]
    assert X.shape[1] == d_in
    Z = np.zeros((T, r), np.float64)
    lib().orc_shared_proj(_p(P, ctypes.c_uint16), _p(X, ctypes.c_uint16), T, d_in, r, _p(Z, ctypes.c_double))
    return Z


def expert_forward(blob: np.ndarray, Z: np.ndarray, ids: np.ndarray, gate_w: np.ndarray,
                   want_experts: bool = True):
    """Returns (Y_e [T][top_k][d_out] or None, Y_sum [T][d_out], status), all fp64."""
    blob = _c(blob, np.uint8)
    E, r, d_out = blob_dims(blob)
    Z = _c(Z, np.float64)
    ids = _c(ids, np.int32)
    g = _c(gate_w, np.float32)
    T, top_k = ids.shape
    assert Z.shape == (T, r) and g.shape == (T, top_k)
    Ys = np.zeros((T, d_out), np.float64)
    Ye = np.zeros((T, top_k, d_out), np.float64) if want_experts else None
    st = ctypes.c_int32(0)
    _check(lib().orc_expert_forward(_p(blob, ctypes.c_uint8), blob.size, _p(Z, ctypes.c_double),
                                    _p(ids, ctypes.c_int32), _p(g, ctypes.c_float), T, top_k,
                                    _p(Ye, ctypes.c_double) if Ye is not None else None,
                                    _p(Ys, ctypes.c_double), ctypes.byref(st)), "expert_forward")
    return Ye, Ys, int(st.value)


def layer_forward(blob_gate, blob_up, phi_t_gate_bits, phi_t_up_bits, x_bits, ids, gate_w, want_experts=True):
    """Both projections of one spectral MoE layer: z = Phi^T x, then the routed experts."""
    out = {}
    for name, blob, phi in (("gate", blob_gate, phi_t_gate_bits), ("up", blob_up, phi_t_up_bits)):
        Z = shared_proj(phi, x_bits)
        Ye, Ys, st = expert_forward(blob, Z, ids, gate_w, want_experts)
        out[name] = {"Z": Z, "Y_experts": Ye, "Y_sum": Ys, "status": st}
    return out


def ffn_down(Y_gate: np.ndarray, Y_up: np.ndarray, w_down_bits: np.ndarray, ids: np.ndarray, gate_w: np.ndarray):
    """Expert FFN output after the gate and up projections (the pages stop at
    gate/up; this is the usual gated expert with a dense fp16 down projection):
    out[t] = sum_s g[t][s] Wd[e] (SiLU(Y_gate[t][s]) * Y_up[t][s]), e = ids[t][s].

    Y_gate, Y_up [T][top_k][d_ff] (fp64), w_down_bits [E][d_model][d_ff] fp16 bits,
    ids [T][top_k], gate_w [T][top_k].  Returns (out [T][d_model] fp64, status)."""
    Yg = _c(Y_gate, np.float64)
    Yu = _c(Y_up, np.float64)
    W = _c(w_down_bits, np.uint16)
    ids = _c(ids, np.int32)
    g = _c(gate_w, np.float32)
    T, top_k = ids.shape
    E, d_model, d_ff = W.shape
    assert Yg.shape == (T, top_k, d_ff) and Yu.shape == Yg.shape and g.shape == ids.shape
    out = np.zeros((T, d_model), np.float64)
    st = ctypes.c_int32(0)
    _check(lib().orc_ffn_down(_p(Yg, ctypes.c_double), _p(Yu, ctypes.c_double), _p(W, ctypes.c_uint16),
                              _p(ids, ctypes.c_int32), _p(g, ctypes.c_float), T, top_k, E, d_model, d_ff,
                              _p(out, ctypes.c_double), ctypes.byref(st)), "ffn_down")
    return out, int(st.value)


def moe_ffn_forward(blob_gate, blob_up, phi_t_gate_bits, phi_t_up_bits, x_bits, ids, gate_w, w_down_bits):
    """The whole expert FFN of one layer: the gate and up projections in spectral
    form (layer_forward), then SiLU(gate) * up and the dense down projection."""
    lf = layer_forward(blob_gate, blob_up, phi_t_gate_bits, phi_t_up_bits, x_bits, ids, gate_w, True)
    out, st = ffn_down(lf["gate"]["Y_experts"], lf["up"]["Y_experts"], w_down_bits, ids, gate_w)
    return out, lf["gate"]["status"] | lf["up"]["status"] | st


def assign_widths(amps: np.ndarray, widths_in_order, counts) -> np.ndarray:
    """Widths [E][r] by descending amplitude within each expert, ties to the lower k:
    the counts[0] largest get widths_in_order[0], the next counts[1] widths_in_order[1], ...
    (the configurations' allocation rule; the pages' allocator chooses the counts)."""
    a = np.asarray(amps, dtype=np.float64)
    E, r = a.shape
    assert sum(int(c) for c in counts) == r
    out = np.zeros((E, r), np.uint8)
    for e in range(E):
        order = sorted(range(r), key=lambda k: (-a[e, k], k))
        pos = 0
        for b, c in zip(widths_in_order, counts):
            for k in order[pos:pos + int(c)]:
                out[e, k] = b
            pos += int(c)
    return out


# ---------------------------------------------------------------------------
# the allocation of widths: FQCM cost and the bit budget (third split, Usage)
# ---------------------------------------------------------------------------
WIDTH_SET = (0, 1, 2, 3, 4, 6, 8, 16)  # the order of the eps arrays


def fqcm_eps(comps: np.ndarray) -> np.ndarray:
    """eps [E][r][8] (fp64): squared error of storing each unit direction at each width
    of WIDTH_SET (the pages' width-dependent distortion, read as ||p - stored p||^2)."""
    comps = _c(comps, np.float32)
    E, r, d_out = comps.shape
    eps = np.zeros((E, r, 8), np.float64)
    _check(lib().orc_fqcm_eps(E, r, d_out, _p(comps, ctypes.c_float), _p(eps, ctypes.c_double)), "fqcm_eps")
    return eps


def fqcm_beta(Z: np.ndarray, ids: np.ndarray, gate_w: np.ndarray, n_experts: int) -> np.ndarray:
    """beta [E][r] (fp64): the activation importance of each spectral direction for each
    expert over calibration tokens, sum over the (token, slot) pairs routed to e of
    g * z_k^2, with z = Phi^T x (third split: beta = phi_k^T X_e G_e X_e^T phi_k)."""
    Z = np.asarray(Z, np.float64)
    ids = np.asarray(ids)
    g = np.asarray(gate_w, np.float64)
    T, r = Z.shape
    beta = np.zeros((n_experts, r), np.float64)
    for t in range(T):
        for j in range(ids.shape[1]):
            e = int(ids[t, j])
            if 0 <= e < n_experts:
                beta[e] += g[t, j] * Z[t] ** 2
    return beta


def allocate_widths(amps: np.ndarray, beta: np.ndarray, eps: np.ndarray, d_out: int, budget_bits: int):
    """Widths [E][r] minimising sum L_{e,k}(b) = a^2 beta eps_b under sum d_out b <= budget_bits
    (the pages: a bit budget, every candidate width of every component considered
    jointly).  Solved as the linear relaxation of this multiple-choice knapsack:
    per component, the lower convex hull of its (bits, loss) points from width 0;
    then every hull segment of every component, in order of loss saved per bit
    (ties: lower component, then earlier segment), taken while it fits; the first
    that does not fit ends the allocation.  A component whose cost is not finite
    at some width keeps width 0.  Returns (widths, total loss)."""
    a = np.asarray(amps, np.float64)
    beta = np.asarray(beta, np.float64)
    eps = np.asarray(eps, np.float64)
    E, r = a.shape
    segs = []
    choice = np.zeros(E * r, np.int64)  # index into WIDTH_SET
    for c in range(E * r):
        e, k = divmod(c, r)
        imp = a[e, k] * a[e, k] * beta[e, k]
        pts = [(d_out * b, imp * eps[e, k, i], i) for i, b in enumerate(WIDTH_SET)]
        if not all(np.isfinite(pt[1]) for pt in pts):
            continue  # a component without a finite cost keeps width 0
        hull = [pts[0]]
        for pt in pts[1:]:
            if pt[1] >= hull[-1][1]:
                continue  # more bits and no less loss
            while len(hull) >= 2:
                A, Bp = hull[-2], hull[-1]
                # Bp leaves the lower hull unless the slope A->Bp is steeper than A->pt
                if (Bp[1] - A[1]) * (pt[0] - A[0]) >= (pt[1] - A[1]) * (Bp[0] - A[0]):
                    hull.pop()
                else:
                    break
            hull.append(pt)
        for s in range(len(hull) - 1):
            gain = hull[s][1] - hull[s + 1][1]
            cost = hull[s + 1][0] - hull[s][0]
            segs.append((gain / cost, c, s, cost, hull[s + 1][2]))
    segs.sort(key=lambda x: (-x[0], x[1], x[2]))
    used = 0
    for eff, c, s, cost, wi in segs:
        if used + cost > budget_bits:
            break
        used += cost
        choice[c] = wi
    widths = np.array([WIDTH_SET[i] for i in choice], np.uint8).reshape(E, r)
    loss = sum(a[c // r, c % r] ** 2 * beta[c // r, c % r] * eps[c // r, c % r, choice[c]] for c in range(E * r))
    return widths, float(loss)


# ---------------------------------------------------------------------------
# offline shared-basis decomposition (used by the reconstruction check)
# ---------------------------------------------------------------------------

def ssd_decompose(W: np.ndarray, rank: int | None = None):
    """Shared-basis spectral decomposition of one projection's experts.

    W: [E][d_out][d_in] expert matrices.  Stacks them vertically into
    W_cat [(E*d_out) x d_in] (so Phi spans the shared input space), takes the
    SVD W_cat = U S Phi^T, sets P = U S and normalises each column of each
    expert's block P_e: a_{e,k} = ||P_e[:,k]||, p_{e,k} = P_e[:,k] / a_{e,k}
    (p = 0 where a = 0).  Keeps the top ``rank`` singular directions.

    Returns (Phi [d_in][rank], a [E][rank], p [E][rank][d_out]) in fp64.
    """
    W = np.asarray(W, dtype=np.float64)
    E, d_out, d_in = W.shape
    rank = d_in if rank is None else rank
    W_cat = W.reshape(E * d_out, d_in)
    U, S, Vt = np.linalg.svd(W_cat, full_matrices=False)
    Phi = Vt[:rank].T
    P = (U[:, :rank] * S[:rank]).reshape(E, d_out, rank)
    a = np.linalg.norm(P, axis=1)  # [E][rank]
    with np.errstate(invalid="ignore", divide="ignore"):
        p = np.where(a[:, None, :] > 0, P / a[:, None, :], 0.0)
    return Phi, a, np.transpose(p, (0, 2, 1)).copy()
