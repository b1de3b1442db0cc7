"""User-facing objects over the C ABI: a packed projection and a spectral MoE
gate/up layer.  torch provides device memory and streams; every computation
is a libbitsmoe kernel."""
from __future__ import annotations

import torch

from . import bitsmoe as B


class PackedProjection:
    """One projection (gate or up) of a spectral MoE layer, packed on the GPU.

    phi_t [r][d_in] fp16 (rows phi_k, kept unquantised), blob = the format-v2
    bit-plane blob of the expert directions, plan = its host descriptor."""

    def __init__(self, plan: B.Plan, blob: torch.Tensor, phi_t: torch.Tensor):
        self.plan, self.blob, self.phi_t = plan, blob, phi_t
        d = plan.dims
        self.d_in, self.d_out, self.n_experts, self.rank, self.top_k = d.d_in, d.d_out, d.n_experts, d.rank, d.top_k

    @classmethod
    def from_factors(cls, phi_t: torch.Tensor, amps: torch.Tensor, comps: torch.Tensor, widths: torch.Tensor,
                     top_k: int, scales: torch.Tensor | None = None, status: torch.Tensor | None = None,
                     stream=None) -> "PackedProjection":
        """Quantise and pack unit directions comps [E][r][d_out] (f32, on the GPU) at
        widths [E][r] (u8) with amplitudes amps [E][r] (f32)."""
        E, r, d_out = comps.shape
        d_in = phi_t.shape[1]
        dev = comps.device
        plan = B.pack_plan(d_in, d_out, E, r, top_k, widths.cpu())
        w_dev = widths.to(dev, torch.uint8).contiguous()
        if scales is None:
            scales = torch.empty((E, r), dtype=torch.int16, device=dev)
            B.compute_scales(plan, comps, w_dev, scales, status, stream)
        blob = torch.empty(plan.blob_bytes, dtype=torch.uint8, device=dev)
        B.pack(plan, comps.contiguous(), w_dev, scales.contiguous(), amps.contiguous(), blob, status, stream)
        return cls(plan, blob, phi_t.contiguous())

    def expert_bytes_touched(self, experts) -> int:
        """Packed bytes (planes + per-component metadata, padding included) of the given experts."""
        h = self.plan.header()
        tot = 0
        for e in experts:
            d = h[64 + 64 * int(e): 128 + 64 * int(e)]
            tot += int(d[8:16].view("uint64")[0])
        return tot


def decompose_and_pack(W: torch.Tensor, rank: int, widths_in_order, counts, top_k: int, status=None,
                       stream=None) -> tuple["PackedProjection", dict]:
    """The offline step before the decode path, on the GPU: the shared-basis spectral
    decomposition of one projection's expert matrices W [E][d_out][d_in] (f32),
    widths by descending amplitude (counts[j] components of each expert at
    widths_in_order[j]), then quantisation and packing.  Returns the packed
    projection and the decomposition (phi_t, sigma, amps, comps, widths)."""
    E, d_out, d_in = W.shape
    dev = W.device
    n = B.ssd_workspace_bytes(E, d_out, d_in, rank)
    if n == 0:
        raise B.BitsMoEError(B.ECUDA, "ssd_workspace_bytes")
    ws = torch.empty(n, dtype=torch.uint8, device=dev)
    phi_t = torch.empty((rank, d_in), dtype=torch.float16, device=dev)
    phi_t32 = torch.empty((rank, d_in), dtype=torch.float32, device=dev)
    sigma = torch.empty(rank, dtype=torch.float32, device=dev)
    amps = torch.empty((E, rank), dtype=torch.float32, device=dev)
    comps = torch.empty((E, rank, d_out), dtype=torch.float32, device=dev)
    B.ssd_decompose(W.contiguous(), rank, phi_t, amps, comps, ws, n, sigma=sigma, phi_t32=phi_t32, status=status,
                    stream=stream)
    del ws
    widths = torch.from_numpy(B.assign_widths(amps.cpu().numpy(), widths_in_order, counts))
    pk = PackedProjection.from_factors(phi_t, amps, comps, widths, top_k, status=status, stream=stream)
    return pk, {"phi_t": phi_t, "phi_t32": phi_t32, "sigma": sigma, "amps": amps, "comps": comps, "widths": widths}


def fqcm_widths(dec: dict, x_calib: torch.Tensor, ids_calib: torch.Tensor, gw_calib: torch.Tensor,
                avg_bits: float, stream=None) -> tuple[torch.Tensor, float, dict]:
    """Widths of one decomposed projection (decompose_and_pack's second result) by the
    FQCM cost under a budget of avg_bits per element: z = Phi^T x of the calibration
    tokens x_calib [T][d_in] fp16 on the GPU, then on the host the activation
    importance beta from z and the routing (ids_calib, gw_calib [T][top_k]), the
    distortion of every component at every width, and the allocation.
    Returns (widths [E][r] u8, total cost, {"beta", "eps"})."""
    phi_t = dec["phi_t"]
    r, d_in = phi_t.shape
    E, _, d_out = dec["comps"].shape
    T = x_calib.shape[0]
    Z = torch.empty((T, r), dtype=torch.float32, device=phi_t.device)
    B.shared_proj(phi_t, x_calib.contiguous(), Z, T, d_in, r, stream)
    beta = B.fqcm_beta(Z.cpu().numpy(), ids_calib.cpu().numpy(), gw_calib.cpu().numpy(), E)
    eps = B.fqcm_eps(dec["comps"].cpu().numpy())
    budget = int(avg_bits * E * r * d_out)
    widths, loss = B.allocate_widths(dec["amps"].cpu().numpy(), beta, eps, d_out, budget)
    return torch.from_numpy(widths), loss, {"beta": beta, "eps": eps}


class SpectralMoELayer:
    """Gate and up projections of one MoE layer in shared-spectral form."""

    def __init__(self, gate: PackedProjection, up: PackedProjection):
        assert gate.d_in == up.d_in and gate.top_k == up.top_k and gate.n_experts == up.n_experts
        self.gate, self.up = gate, up
        self._ws = {}
        self._ios = {}

    def workspace(self, T: int) -> torch.Tensor:
        """The layer's workspace for T tokens, allocated on first use.  The plans
        are immutable, so its size for a given T never changes."""
        ws = self._ws.get(T)
        if ws is None:
            n = B.layer_workspace_bytes(self.gate.plan, self.up.plan, T)
            # zero-filled once: its head keeps the fused path's counters between calls
            ws = torch.zeros(max(n, 256), dtype=torch.uint8, device=self.gate.blob.device)
            self._ws[T] = ws
        return ws

    def _proj_ios(self, out: dict) -> tuple:
        """The two projections' I/O descriptors for these output buffers, reused
        while a caller keeps passing the same buffers (a decode loop)."""
        key = tuple(None if t is None else t.data_ptr()
                    for t in (out["Y_sum_gate"], out["Y_sum_up"], out.get("Z_gate"), out.get("Z_up"),
                              out.get("Y_experts_gate"), out.get("Y_experts_up")))
        ios = self._ios.get(key)
        if ios is None:
            ios = tuple(B.proj_io(p.plan, p.blob, p.phi_t, out[f"Y_sum_{name}"], out.get(f"Z_{name}"),
                                  out.get(f"Y_experts_{name}"))
                        for name, p in (("gate", self.gate), ("up", self.up)))
            if len(self._ios) >= 64:
                self._ios.clear()
            self._ios[key] = ios
        return ios

    def forward(self, x: torch.Tensor, topk_ids: torch.Tensor, gate_w: torch.Tensor, out: dict | None = None,
                want_experts: bool = False, want_z: bool = False, status: torch.Tensor | None = None,
                stream=None, next_layer: "SpectralMoELayer | None" = None) -> dict:
        """x [T][d_in] fp16, topk_ids [T][top_k] int32, gate_w [T][top_k] f32 (all on the GPU).
        Returns Y_sum_gate / Y_sum_up [T][d_out] f32 (and Y_experts_* / Z_* on request).
        next_layer: the layer a decode loop runs next; its Phi^T are prefetched into
        L2 while this call evaluates its experts (single-token path)."""
        T = x.shape[0]
        dev = x.device
        if out is None:
            out = {}
            for name, p in (("gate", self.gate), ("up", self.up)):
                out[f"Y_sum_{name}"] = torch.empty((T, p.d_out), dtype=torch.float32, device=dev)
                if want_experts:
                    out[f"Y_experts_{name}"] = torch.empty((T, p.top_k, p.d_out), dtype=torch.float32, device=dev)
                if want_z:
                    out[f"Z_{name}"] = torch.empty((T, p.rank), dtype=torch.float32, device=dev)
        ios = self._proj_ios(out)
        ws = self.workspace(T)
        if next_layer is None:
            B.layer_forward(ios[0], ios[1], x, topk_ids, gate_w, T, ws, ws.numel(), status, stream)
        else:
            B.layer_forward_chained(ios[0], ios[1], x, topk_ids, gate_w, T, ws, ws.numel(), next_layer.gate.phi_t,
                                    next_layer.up.phi_t, status, stream)
        return out


class SpectralMoEFFN:
    """A routed expert FFN: the gate and up projections in shared-spectral form
    (SpectralMoELayer), then SiLU(gate) * up and a dense fp16 down projection per
    expert, summed over each token's slots with its gate weights -- one
    bitsmoe_ffn_forward call.

    w_down [E][d_model][d_ff] fp16 on the GPU, d_model = the layer's d_in and
    d_ff = the gate/up d_out."""

    def __init__(self, layer: SpectralMoELayer, w_down: torch.Tensor):
        g = layer.gate
        assert layer.up.d_out == g.d_out
        assert w_down.dtype == torch.float16 and tuple(w_down.shape) == (g.n_experts, g.d_in, g.d_out)
        self.layer = layer
        self.w_down = w_down.contiguous()
        self.dims = B.ffn_dims(g.d_in, g.d_out, g.n_experts, g.top_k)
        self._ws = {}

    def workspace(self, T: int) -> torch.Tensor:
        """The call's workspace for T tokens (the layer's, then the down step's),
        zero-filled once on first use: its head keeps the fused path's counters."""
        ws = self._ws.get(T)
        if ws is None:
            n = B.ffn_workspace_bytes(self.layer.gate.plan, self.layer.up.plan, T)
            ws = torch.zeros(max(n, 256), dtype=torch.uint8, device=self.w_down.device)
            self._ws[T] = ws
        return ws

    def launches(self, T: int) -> int:
        """Kernels one forward launches for T tokens (the layer's, then the down step's)."""
        return B.ffn_launches(self.layer.gate.plan, self.layer.up.plan, T)

    def gate_up_buffers(self, T: int, device) -> dict:
        """Output buffers of the gate and up projections (routed sums and per-slot outputs)."""
        out = {}
        for name, p in (("gate", self.layer.gate), ("up", self.layer.up)):
            out[f"Y_sum_{name}"] = torch.empty((T, p.d_out), dtype=torch.float32, device=device)
            out[f"Y_experts_{name}"] = torch.empty((T, p.top_k, p.d_out), dtype=torch.float32, device=device)
        return out

    def forward(self, x: torch.Tensor, topk_ids: torch.Tensor, gate_w: torch.Tensor, out: torch.Tensor | None = None,
                gate_up: dict | None = None, status: torch.Tensor | None = None, stream=None) -> torch.Tensor:
        """x [T][d_in] fp16, topk_ids [T][top_k] int32, gate_w [T][top_k] f32 -> out [T][d_model] f32.
        gate_up: the gate/up output buffers (gate_up_buffers) to reuse between calls."""
        T = x.shape[0]
        if out is None:
            out = torch.empty((T, self.dims.d_model), dtype=torch.float32, device=x.device)
        if gate_up is None:
            gate_up = self.gate_up_buffers(T, x.device)
        ios = self.layer._proj_ios(gate_up)
        ws = self.workspace(T)
        B.ffn_forward(ios[0], ios[1], self.w_down, x, topk_ids, gate_w, T, out, ws, ws.numel(), status, stream)
        return out
