"""ctypes binding of libbitsmoe (include/bitsmoe.h), same names as the C calls.

Argument marshalling only: every step of the path runs in the library's CUDA
kernels.  Tensors are torch tensors on the GPU (device pointers are taken with
``data_ptr()``); the stream defaults to torch's current stream.  If the shared
library is missing the import of any call raises: there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np
import torch

# BITSMOE_CHECKED=1 selects the bounds-checked build (libbitsmoe_checked.so): every
# computed index of the expert kernels is checked, a violation sets ST_BOUNDS.
_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)),
                         "libbitsmoe_checked.so" if os.environ.get("BITSMOE_CHECKED") == "1" else "libbitsmoe.so")

OK, EINVAL, EWIDTH, ESIZE, ECUDA, EFORMAT, ENOMEM = 0, -1, -2, -3, -4, -5, -6
ST_NONFINITE, ST_BADSCALE, ST_BADEXPERT, ST_TIMEOUT, ST_PLANMISMATCH, ST_BOUNDS = 1, 2, 4, 8, 16, 32
ST_NOCONVERGE = 64

# Every symbol include/bitsmoe.h declares.
EXPORTS = (
    "bitsmoe_pack_plan", "bitsmoe_plan_from_header", "bitsmoe_plan_free", "bitsmoe_plan_blob_bytes",
    "bitsmoe_plan_header_bytes", "bitsmoe_plan_get_dims", "bitsmoe_plan_write_header", "bitsmoe_compute_scales",
    "bitsmoe_pack", "bitsmoe_unpack_q", "bitsmoe_shared_proj", "bitsmoe_expert_workspace_bytes",
    "bitsmoe_expert_forward", "bitsmoe_layer_workspace_bytes", "bitsmoe_layer_launches", "bitsmoe_layer_forward",
    "bitsmoe_layer_forward_chained", "bitsmoe_layer_forward_t1_noalloc", "bitsmoe_ffn_down_workspace_bytes",
    "bitsmoe_ffn_down_launches", "bitsmoe_ffn_down", "bitsmoe_ffn_workspace_bytes", "bitsmoe_ffn_launches",
    "bitsmoe_ffn_forward", "bitsmoe_ssd_workspace_bytes", "bitsmoe_ssd_decompose", "bitsmoe_assign_widths",
    "bitsmoe_fqcm_eps", "bitsmoe_fqcm_beta", "bitsmoe_allocate_widths",
    "bitsmoe_read_status", "bitsmoe_strerror", "bitsmoe_version",
)


class BitsMoEError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {strerror(code)} ({code})")
        self.code = code


class Dims(ctypes.Structure):
    _fields_ = [("d_in", ctypes.c_int32), ("d_out", ctypes.c_int32), ("n_experts", ctypes.c_int32),
                ("rank", ctypes.c_int32), ("top_k", ctypes.c_int32)]


class FfnDims(ctypes.Structure):
    _fields_ = [("d_model", ctypes.c_int32), ("d_ff", ctypes.c_int32), ("n_experts", ctypes.c_int32),
                ("top_k", ctypes.c_int32)]


class ProjIO(ctypes.Structure):
    _fields_ = [("plan", ctypes.c_void_p), ("blob", ctypes.c_void_p), ("phi_t", ctypes.c_void_p),
                ("Z", ctypes.c_void_p), ("Y_experts", ctypes.c_void_p), ("Y_sum", ctypes.c_void_p)]


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded library; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(f"{_LIB_PATH} is missing: build it with mixed_precision_decode_b200.build.build()"
                               f" (checked=True for the bounds-checked build)")
        L = ctypes.CDLL(_LIB_PATH)
        vp, u64, i32 = ctypes.c_void_p, ctypes.c_uint64, ctypes.c_int32
        sig = {
            "bitsmoe_pack_plan": ([ctypes.POINTER(Dims), vp, ctypes.POINTER(vp)], ctypes.c_int),
            "bitsmoe_plan_from_header": ([vp, u64, i32, i32, ctypes.POINTER(vp)], ctypes.c_int),
            "bitsmoe_plan_free": ([vp], None),
            "bitsmoe_plan_blob_bytes": ([vp], u64),
            "bitsmoe_plan_header_bytes": ([vp], u64),
            "bitsmoe_plan_get_dims": ([vp, ctypes.POINTER(Dims)], ctypes.c_int),
            "bitsmoe_plan_write_header": ([vp, vp, u64], ctypes.c_int),
            "bitsmoe_compute_scales": ([vp, vp, vp, vp, vp, vp], ctypes.c_int),
            "bitsmoe_pack": ([vp, vp, vp, vp, vp, vp, vp, vp], ctypes.c_int),
            "bitsmoe_unpack_q": ([vp, vp, vp, vp], ctypes.c_int),
            "bitsmoe_shared_proj": ([vp, vp, vp, i32, i32, i32, vp], ctypes.c_int),
            "bitsmoe_expert_workspace_bytes": ([vp, i32], u64),
            "bitsmoe_expert_forward": ([vp, vp, vp, vp, vp, i32, vp, vp, vp, u64, vp, vp], ctypes.c_int),
            "bitsmoe_layer_workspace_bytes": ([vp, vp, i32], u64),
            "bitsmoe_layer_launches": ([vp, vp, i32], ctypes.c_int),
            "bitsmoe_layer_forward": ([ctypes.POINTER(ProjIO), ctypes.POINTER(ProjIO), vp, vp, vp, i32, vp, u64,
                                       vp, vp], ctypes.c_int),
            "bitsmoe_layer_forward_chained": ([ctypes.POINTER(ProjIO), ctypes.POINTER(ProjIO), vp, vp, vp, i32, vp,
                                               u64, vp, vp, vp, vp], ctypes.c_int),
            "bitsmoe_layer_forward_t1_noalloc": ([ctypes.POINTER(ProjIO), ctypes.POINTER(ProjIO), vp, vp, vp, vp,
                                                  vp], ctypes.c_int),
            "bitsmoe_ffn_down_workspace_bytes": ([ctypes.POINTER(FfnDims), i32], u64),
            "bitsmoe_ffn_down_launches": ([ctypes.POINTER(FfnDims), i32], ctypes.c_int),
            "bitsmoe_ffn_down": ([ctypes.POINTER(FfnDims), vp, vp, vp, vp, vp, i32, vp, vp, u64, vp, vp],
                                 ctypes.c_int),
            "bitsmoe_ffn_workspace_bytes": ([vp, vp, i32], u64),
            "bitsmoe_ffn_launches": ([vp, vp, i32], ctypes.c_int),
            "bitsmoe_ffn_forward": ([ctypes.POINTER(ProjIO), ctypes.POINTER(ProjIO), vp, vp, vp, vp, i32, vp, vp, u64,
                                     vp, vp], ctypes.c_int),
            "bitsmoe_ssd_workspace_bytes": ([i32, i32, i32, i32], u64),
            "bitsmoe_ssd_decompose": ([vp, i32, i32, i32, i32, vp, vp, vp, vp, vp, vp, u64, vp, vp], ctypes.c_int),
            "bitsmoe_assign_widths": ([vp, i32, i32, vp, vp, i32, vp], ctypes.c_int),
            "bitsmoe_fqcm_eps": ([vp, i32, i32, i32, vp], ctypes.c_int),
            "bitsmoe_fqcm_beta": ([vp, vp, vp, i32, i32, i32, i32, vp], ctypes.c_int),
            "bitsmoe_allocate_widths": ([vp, vp, vp, i32, i32, i32, u64, vp, vp], ctypes.c_int),
            "bitsmoe_read_status": ([vp, vp, ctypes.POINTER(ctypes.c_int32)], ctypes.c_int),
            "bitsmoe_strerror": ([ctypes.c_int], ctypes.c_char_p),
            "bitsmoe_version": ([], ctypes.c_int),
        }
        for name, (args, res) in sig.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = res
        _lib = L
    return _lib


def strerror(code: int) -> str:
    return lib().bitsmoe_strerror(code).decode()


def version() -> int:
    return lib().bitsmoe_version()


def _check(rc: int, what: str):
    if rc != 0:
        raise BitsMoEError(rc, what)


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, torch.Tensor):
        return t.data_ptr()
    return int(t)


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else None
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


class Plan:
    """Owns one bitsmoe_plan (host object describing one projection's blob)."""

    def __init__(self, handle: int):
        self._h = ctypes.c_void_p(handle)

    @property
    def handle(self) -> ctypes.c_void_p:
        return self._h

    def __del__(self):
        if getattr(self, "_h", None) is not None and self._h.value and _lib is not None:
            _lib.bitsmoe_plan_free(self._h)
            self._h = None

    @property
    def blob_bytes(self) -> int:
        return int(lib().bitsmoe_plan_blob_bytes(self._h))

    @property
    def header_bytes(self) -> int:
        return int(lib().bitsmoe_plan_header_bytes(self._h))

    @property
    def dims(self) -> Dims:
        d = Dims()
        _check(lib().bitsmoe_plan_get_dims(self._h, ctypes.byref(d)), "plan_get_dims")
        return d

    def header(self) -> np.ndarray:
        out = np.zeros(self.header_bytes, np.uint8)
        _check(lib().bitsmoe_plan_write_header(self._h, out.ctypes.data, out.size), "plan_write_header")
        return out


def pack_plan(d_in: int, d_out: int, n_experts: int, rank: int, top_k: int, widths) -> Plan:
    w = np.ascontiguousarray(widths.cpu().numpy() if isinstance(widths, torch.Tensor) else widths, dtype=np.uint8)
    d = Dims(d_in, d_out, n_experts, rank, top_k)
    h = ctypes.c_void_p()
    _check(lib().bitsmoe_pack_plan(ctypes.byref(d), w.ctypes.data, ctypes.byref(h)), "pack_plan")
    return Plan(h.value)


def plan_from_header(header, d_in: int, top_k: int) -> Plan:
    hb = np.ascontiguousarray(header.cpu().numpy() if isinstance(header, torch.Tensor) else header, dtype=np.uint8)
    h = ctypes.c_void_p()
    _check(lib().bitsmoe_plan_from_header(hb.ctypes.data, hb.size, d_in, top_k, ctypes.byref(h)), "plan_from_header")
    return Plan(h.value)


def compute_scales(plan: Plan, comps, widths, scales, status=None, stream=None):
    _check(lib().bitsmoe_compute_scales(plan.handle, _ptr(comps), _ptr(widths), _ptr(scales), _ptr(status),
                                        _stream(stream)), "compute_scales")


def pack(plan: Plan, comps, widths, scales, amps, blob, status=None, stream=None):
    _check(lib().bitsmoe_pack(plan.handle, _ptr(comps), _ptr(widths), _ptr(scales), _ptr(amps), _ptr(blob),
                              _ptr(status), _stream(stream)), "pack")


def unpack_q(plan: Plan, blob, q, stream=None):
    _check(lib().bitsmoe_unpack_q(plan.handle, _ptr(blob), _ptr(q), _stream(stream)), "unpack_q")


def shared_proj(phi_t, X, Z, T: int, d_in: int, r: int, stream=None):
    _check(lib().bitsmoe_shared_proj(_ptr(phi_t), _ptr(X), _ptr(Z), T, d_in, r, _stream(stream)), "shared_proj")


def expert_workspace_bytes(plan: Plan, T: int) -> int:
    return int(lib().bitsmoe_expert_workspace_bytes(plan.handle, T))


def expert_forward(plan: Plan, blob, Z, topk_ids, gate_w, T: int, Y_experts, Y_sum, workspace, workspace_bytes: int,
                   status=None, stream=None):
    _check(lib().bitsmoe_expert_forward(plan.handle, _ptr(blob), _ptr(Z), _ptr(topk_ids), _ptr(gate_w), T,
                                        _ptr(Y_experts), _ptr(Y_sum), _ptr(workspace), workspace_bytes,
                                        _ptr(status), _stream(stream)), "expert_forward")


def layer_workspace_bytes(plan_gate: Plan, plan_up: Plan, T: int) -> int:
    return int(lib().bitsmoe_layer_workspace_bytes(plan_gate.handle, plan_up.handle, T))


def layer_launches(plan_gate: Plan, plan_up: Plan, T: int) -> int:
    n = int(lib().bitsmoe_layer_launches(plan_gate.handle, plan_up.handle, T))
    if n < 0:
        raise BitsMoEError(n, "layer_launches")
    return n


def proj_io(plan: Plan, blob, phi_t, Y_sum, Z=None, Y_experts=None) -> ProjIO:
    return ProjIO(plan.handle.value, _ptr(blob), _ptr(phi_t), _ptr(Z), _ptr(Y_experts), _ptr(Y_sum))


def layer_forward(gate: ProjIO, up: ProjIO, X, topk_ids, gate_w, T: int, workspace, workspace_bytes: int,
                  status=None, stream=None):
    _check(lib().bitsmoe_layer_forward(ctypes.byref(gate), ctypes.byref(up), _ptr(X), _ptr(topk_ids), _ptr(gate_w),
                                       T, _ptr(workspace), workspace_bytes, _ptr(status), _stream(stream)),
           "layer_forward")


def layer_forward_chained(gate: ProjIO, up: ProjIO, X, topk_ids, gate_w, T: int, workspace, workspace_bytes: int,
                          next_phi_t_gate, next_phi_t_up, status=None, stream=None):
    _check(lib().bitsmoe_layer_forward_chained(ctypes.byref(gate), ctypes.byref(up), _ptr(X), _ptr(topk_ids),
                                               _ptr(gate_w), T, _ptr(workspace), workspace_bytes,
                                               _ptr(next_phi_t_gate), _ptr(next_phi_t_up), _ptr(status),
                                               _stream(stream)),
           "layer_forward_chained")


def layer_forward_t1_noalloc(gate: ProjIO, up: ProjIO, X, topk_ids, gate_w, status=None, stream=None):
    _check(lib().bitsmoe_layer_forward_t1_noalloc(ctypes.byref(gate), ctypes.byref(up), _ptr(X), _ptr(topk_ids),
                                                  _ptr(gate_w), _ptr(status), _stream(stream)),
           "layer_forward_t1_noalloc")


def ffn_dims(d_model: int, d_ff: int, n_experts: int, top_k: int) -> FfnDims:
    return FfnDims(d_model, d_ff, n_experts, top_k)


def ffn_down_workspace_bytes(dims: FfnDims, T: int) -> int:
    return int(lib().bitsmoe_ffn_down_workspace_bytes(ctypes.byref(dims), T))


def ffn_down_launches(dims: FfnDims, T: int) -> int:
    n = int(lib().bitsmoe_ffn_down_launches(ctypes.byref(dims), T))
    if n < 0:
        raise BitsMoEError(n, "ffn_down_launches")
    return n


def ffn_down(dims: FfnDims, w_down, Y_gate, Y_up, topk_ids, gate_w, T: int, out, workspace=None,
             workspace_bytes: int = 0, status=None, stream=None):
    _check(lib().bitsmoe_ffn_down(ctypes.byref(dims), _ptr(w_down), _ptr(Y_gate), _ptr(Y_up), _ptr(topk_ids),
                                  _ptr(gate_w), T, _ptr(out), _ptr(workspace), workspace_bytes, _ptr(status),
                                  _stream(stream)), "ffn_down")


def ffn_workspace_bytes(plan_gate: Plan, plan_up: Plan, T: int) -> int:
    return int(lib().bitsmoe_ffn_workspace_bytes(plan_gate.handle, plan_up.handle, T))


def ffn_launches(plan_gate: Plan, plan_up: Plan, T: int) -> int:
    n = int(lib().bitsmoe_ffn_launches(plan_gate.handle, plan_up.handle, T))
    if n < 0:
        raise BitsMoEError(n, "ffn_launches")
    return n


def ffn_forward(gate: ProjIO, up: ProjIO, w_down, X, topk_ids, gate_w, T: int, out, workspace, workspace_bytes: int,
                status=None, stream=None):
    _check(lib().bitsmoe_ffn_forward(ctypes.byref(gate), ctypes.byref(up), _ptr(w_down), _ptr(X), _ptr(topk_ids),
                                     _ptr(gate_w), T, _ptr(out), _ptr(workspace), workspace_bytes, _ptr(status),
                                     _stream(stream)), "ffn_forward")


def ssd_workspace_bytes(n_experts: int, d_out: int, d_in: int, rank: int) -> int:
    return int(lib().bitsmoe_ssd_workspace_bytes(n_experts, d_out, d_in, rank))


def ssd_decompose(W, rank: int, phi_t, amps, comps, workspace, workspace_bytes: int, sigma=None, phi_t32=None,
                  status=None, stream=None):
    """W [E][d_out][d_in] f32 (GPU) -> phi_t [rank][d_in] fp16, amps [E][rank], comps [E][rank][d_out]."""
    E, d_out, d_in = W.shape
    _check(lib().bitsmoe_ssd_decompose(_ptr(W), E, d_out, d_in, rank, _ptr(phi_t), _ptr(phi_t32), _ptr(sigma),
                                       _ptr(amps), _ptr(comps), _ptr(workspace), workspace_bytes, _ptr(status),
                                       _stream(stream)),
           "ssd_decompose")


def assign_widths(amps_host, widths_in_order, counts) -> np.ndarray:
    """Widths [E][r] u8 by descending amplitude within each expert (host)."""
    a = np.ascontiguousarray(np.asarray(amps_host, dtype=np.float32))
    E, r = a.shape
    wo = np.ascontiguousarray(np.asarray(widths_in_order, dtype=np.uint8))
    ct = np.ascontiguousarray(np.asarray(counts, dtype=np.int32))
    out = np.zeros((E, r), np.uint8)
    _check(lib().bitsmoe_assign_widths(a.ctypes.data, E, r, wo.ctypes.data, ct.ctypes.data, len(wo), out.ctypes.data),
           "assign_widths")
    return out


WIDTH_SET = (0, 1, 2, 3, 4, 6, 8, 16)  # the width order of eps arrays


def _host(a, dtype):
    return np.ascontiguousarray(np.asarray(a, dtype=dtype))


def fqcm_eps(comps_host) -> np.ndarray:
    """eps [E][r][8] f64: squared error of each unit direction stored at each width."""
    c = _host(comps_host, np.float32)
    E, r, d_out = c.shape
    out = np.zeros((E, r, 8), np.float64)
    _check(lib().bitsmoe_fqcm_eps(c.ctypes.data, E, r, d_out, out.ctypes.data), "fqcm_eps")
    return out


def fqcm_beta(Z_host, topk_ids_host, gate_w_host, n_experts: int) -> np.ndarray:
    """beta [E][r] f64 from z = Phi^T x of calibration tokens and their routing."""
    Z = _host(Z_host, np.float32)
    ids = _host(topk_ids_host, np.int32)
    g = _host(gate_w_host, np.float32)
    T, r = Z.shape
    out = np.zeros((n_experts, r), np.float64)
    _check(lib().bitsmoe_fqcm_beta(Z.ctypes.data, ids.ctypes.data, g.ctypes.data, T, ids.shape[1], n_experts, r,
                                   out.ctypes.data), "fqcm_beta")
    return out


def allocate_widths(amps_host, beta_host, eps_host, d_out: int, budget_bits: int) -> tuple[np.ndarray, float]:
    """(widths [E][r] u8, total cost) under sum d_out b <= budget_bits."""
    a = _host(amps_host, np.float32)
    b = _host(beta_host, np.float64)
    e = _host(eps_host, np.float64)
    E, r = a.shape
    w = np.zeros((E, r), np.uint8)
    loss = ctypes.c_double(0.0)
    _check(lib().bitsmoe_allocate_widths(a.ctypes.data, b.ctypes.data, e.ctypes.data, E, r, d_out, int(budget_bits),
                                         w.ctypes.data, ctypes.byref(loss)), "allocate_widths")
    return w, float(loss.value)


def read_status(status, stream=None) -> int:
    out = ctypes.c_int32(0)
    _check(lib().bitsmoe_read_status(_ptr(status), _stream(stream), ctypes.byref(out)), "read_status")
    return int(out.value)
