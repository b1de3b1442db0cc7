#!/usr/bin/env python
"""Decode throughput of the spectral MoE gate/up forward (BitsMoE) on B200.

One step = one layer forward (gate and up projections: z = Phi^T x for both,
the routed bit-plane experts of both, their routed sums) for one batch of
decode tokens.  Default workload: the Qwen3-30B-A3B-shaped layer (d_in 2048,
d_out 768, 128 experts, top-8, rank 2048, ~2.08 bits) at one token per step.

Steps rotate over distinct layer copies whose bytes exceed L2 several times,
each with its own pre-drawn token and routing, all resident in HBM before the
timed region; the K timed steps are CUDA-graph replays timed with CUDA events
on the launching stream (max over ranks).  Prints one JSON line on rank 0.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
"""
from __future__ import annotations

import argparse
import json
import math
import os
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode tokens/s and HBM GB/s (% of B200 roofline), spectral MoE gate/up fwd"
FALLBACK_HBM_GBS = 6650.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=2000)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", default="qwen_t1")
    ap.add_argument("--tokens", type=int, default=None, help="override tokens per step")
    ap.add_argument("--layers", type=int, default=16, help="distinct layer copies rotated through")
    ap.add_argument("--graph-steps", type=int, default=1000)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-chained", action="store_true", help="skip the chained-loop measurement")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--ffn", action="store_true",
                    help="time the whole expert FFN step instead (gate/up layer, then SiLU(gate)*up and the dense "
                         "fp16 down projection), with the down kernel's own roofline")
    ap.add_argument("--ffn-two-calls", action="store_true",
                    help="with --ffn: run each step as bitsmoe_layer_forward then bitsmoe_ffn_down")
    ap.add_argument("--ssd", action="store_true",
                    help="time the offline step instead: the shared-basis decomposition of one projection's experts, "
                         "widths by descending amplitude, quantisation and packing")
    ap.add_argument("--fqcm", action="store_true",
                    help="with --ssd: choose the widths by the FQCM cost under the configuration's average bits "
                         "(calibration: --calib-tokens seeded tokens and routings) instead of its fixed fractions")
    ap.add_argument("--calib-tokens", type=int, default=4096)
    ap.add_argument("--clock-window", type=float, default=0.25,
                    help="seconds of untimed replays of the same loop before the timed steps, during which (and "
                         "during the timed steps) the SM clock is sampled")
    return ap.parse_args()


# ---------------------------------------------------------------------------
# distributed plumbing (one process per GPU; timing only, no data exchange)
# ---------------------------------------------------------------------------
class Dist:
    def __init__(self, gpus: int):
        import torch
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = None
        if self.world > 1:
            import datetime
            import torch.distributed as dist
            backend = "nccl" if torch.cuda.is_available() else "gloo"
            if backend == "nccl":
                torch.cuda.set_device(self.local)
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
            self.pg = dist
        elif torch.cuda.is_available():
            torch.cuda.set_device(0)

    def barrier(self):
        if self.pg:
            self.pg.barrier()

    def max(self, v: float) -> float:
        if not self.pg:
            return v
        import torch
        dev = "cuda" if torch.cuda.is_available() else "cpu"
        t = torch.tensor([v], dtype=torch.float64, device=dev)
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg:
            self.pg.destroy_process_group()


# ---------------------------------------------------------------------------
# workload
# ---------------------------------------------------------------------------
def algorithmic_bytes(cfg, counts, ids_step, T) -> dict:
    """Bytes the method must move for one layer step: Phi (both projections,
    fp16), the packed planes and per-component metadata (idx u16, scale fp16,
    amp f32) of each distinct routed expert (no padding), x, routing, outputs."""
    import numpy as np
    phi = 2 * cfg.d_in * cfg.rank * 2
    experts = np.unique(ids_step.reshape(-1))
    planes = meta = 0
    for proj in ("gate", "up"):
        c = counts[proj]  # [E][8]: n_b for b = 16,8,6,4,3,2,1 and zero
        for e in experts:
            n = c[int(e)]
            bits = 16 * n[0] + 8 * n[1] + 6 * n[2] + 4 * n[3] + 3 * n[4] + 2 * n[5] + 1 * n[6]
            planes += cfg.d_out * int(bits) // 8
            meta += int(n[1:7].sum()) * 8 + int(n[0]) * 6
    act = T * cfg.d_in * 2 + T * cfg.top_k * 8 + 2 * T * cfg.d_out * 4
    return {"phi": phi, "planes": planes, "meta": meta, "act": act, "total": phi + planes + meta + act,
            "distinct_experts": int(len(experts))}


def lds_wavefronts(cfg, counts, ids_step, T) -> int:
    """Shared-memory wavefronts (128 B each) of the multi-token expert kernel's
    table lookups for one layer step.  Per distinct routed expert and token group
    of up to 4 of its tokens, every plane word (bit planes of 32 members, padded)
    is looked up in every 32-row tile: one 4-byte lookup per 4 bits (8 wavefronts
    per warp) for a one-token group, else two 8-byte lookups per 4 bits for each
    token pair (16 wavefronts per pair)."""
    import numpy as np
    tiles = (cfg.d_out + 31) // 32
    ids = ids_step.reshape(-1)
    experts, per_expert = np.unique(ids, return_counts=True)
    widths = (8, 6, 4, 3, 2, 1)  # the bit-plane groups, storage order after fp16
    total = 0
    for proj in ("gate", "up"):
        c = counts[proj]
        for e, te in zip(experts, per_expert):
            n = c[int(e)]
            pw = sum(b * ((int(n[g + 1]) + 31) // 32) for g, b in enumerate(widths))
            groups = [4] * (int(te) // 4) + ([int(te) % 4] if int(te) % 4 else [])
            per_tile = sum(8 if nt == 1 else 16 * ((nt + 1) // 2) for nt in groups)
            total += pw * tiles * per_tile
    return total


def lds_peak_gbs(sm_mhz: float, sms: int = 148) -> float:
    """Shared-memory bandwidth from the unit counts: 128 B per clock per SM."""
    return 128.0 * sms * sm_mhz * 1e6 / 1e9


def plan_counts(plan) -> "np.ndarray":
    import numpy as np
    h = plan.header()
    E = plan.dims.n_experts
    out = np.zeros((E, 8), np.int64)
    for e in range(E):
        out[e] = h[64 + 64 * e + 44: 64 + 64 * e + 60].view(np.uint16)
    return out


class Workload:
    """L distinct packed layers + G pre-drawn (x, ids, gate_w) steps, on one GPU."""

    def __init__(self, cfg, n_layers, n_steps, seed_base, keep_comps_of_layer0=False):
        import torch
        from mixed_precision_decode_b200 import synth
        from mixed_precision_decode_b200.layer import PackedProjection, SpectralMoELayer
        self.cfg = cfg
        dev = torch.device("cuda")
        self.layers, self.counts, self.host0 = [], [], None
        for l in range(n_layers):
            gen = synth.make_generator(seed_base + l, dev)
            projs, counts, host = {}, {}, {}
            for name in ("gate", "up"):
                P = synth.make_projection(cfg, gen, dev)
                projs[name] = PackedProjection.from_factors(P["phi_t"], P["amps"], P["comps"], P["widths"], cfg.top_k)
                counts[name] = plan_counts(projs[name].plan)
                if keep_comps_of_layer0 and l == 0:
                    host[name] = {"phi_t": P["phi_t"], "amps": P["amps"], "widths": P["widths"], "comps": P["comps"]}
                del P
            self.layers.append(SpectralMoELayer(projs["gate"], projs["up"]))
            self.counts.append(counts)
            if host:
                self.host0 = host
        torch.cuda.synchronize()
        T = cfg.tokens
        gen = synth.make_generator(seed_base + 999_983, dev)
        self.x = torch.randn((n_steps, T, cfg.d_in), generator=gen, device=dev).to(torch.float16)
        ids, gw = [], []
        for s in range(n_steps):
            i, w = synth.make_routing(cfg, gen, dev, T)
            ids.append(i)
            gw.append(w)
        self.ids = torch.stack(ids).contiguous()
        self.gw = torch.stack(gw).contiguous()
        self.out = [layer.forward(self.x[0], self.ids[0], self.gw[0]) for layer in self.layers]
        self.n_steps = n_steps
        torch.cuda.synchronize()

    def layer_of(self, s):
        return s % len(self.layers)

    def data_of(self, s):
        return s % self.n_steps

    def step(self, s, stream=None, next_s=None):
        """Step s of the decode loop (any integer): layer s mod L on pre-drawn
        token and routing s mod n_steps.  With next_s, as a decode loop that runs
        step next_s after it (its layer's Phi^T is prefetched while this step
        evaluates experts)."""
        l, d = self.layer_of(s), self.data_of(s)
        nxt = None if next_s is None else self.layers[self.layer_of(next_s)]
        self.layers[l].forward(self.x[d], self.ids[d], self.gw[d], out=self.out[l], stream=stream, next_layer=nxt)

    def blob_bytes_total(self):
        return sum(L.gate.blob.numel() + L.up.blob.numel() + 2 * L.gate.phi_t.numel() * 2 for L in self.layers) // 2 * 2


# ---------------------------------------------------------------------------
# clocks during the timed region (NVML reads only)
# ---------------------------------------------------------------------------
class ClockSampler:
    """SM clock and clock-event reasons from NVML (reads only; no GPU setting is
    changed).  A thread polls while the sampler is entered; `sample_now()` adds
    one sample from the calling thread.  With `timed_events` = (ev0, ev1) set,
    the poll thread spins without sleeping while ev0 has completed and ev1 has
    not, and counts those samples as taken inside the timed region."""
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x2: "applications_clocks_setting", 0x1: "gpu_idle"}

    def __init__(self, index: int, period_s: float = 0.001):
        self.ok = False
        self.period = period_s
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = self._handle(pynvml, index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self._get_r = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                pynvml.nvmlDeviceGetCurrentClocksThrottleReasons
            self.ok = True
        except Exception as e:  # no NVML: report that instead of clocks
            self.err = str(e)
        self.samples, self.timed_samples, self.reasons = [], [], 0
        self.timed_events = None
        self._lock = threading.Lock()
        self._stop = threading.Event()

    @staticmethod
    def _handle(nv, index: int):
        """NVML handle of CUDA device `index`, matched by UUID (NVML numbers every GPU
        of the host; CUDA only the visible ones), else by index."""
        try:
            import torch
            u = str(torch.cuda.get_device_properties(index).uuid)
            u = u if u.startswith("GPU-") else "GPU-" + u
            return nv.nvmlDeviceGetHandleByUUID(u)
        except Exception:
            return nv.nvmlDeviceGetHandleByIndex(index)

    def sample_now(self, in_timed: bool = False):
        if not self.ok:
            return
        try:
            mhz = self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)
            r = int(self._get_r(self.h))
        except Exception:
            return
        with self._lock:
            self.samples.append(mhz)
            if in_timed:
                self.timed_samples.append(mhz)
            self.reasons |= r

    def _in_timed(self) -> bool:
        ev = self.timed_events
        if ev is None:
            return False
        try:
            return bool(ev[0].query()) and not bool(ev[1].query())
        except Exception:
            return False

    def _run(self):
        while not self._stop.is_set():
            inside = self._in_timed()
            self.sample_now(inside)
            if not inside:
                time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "error": getattr(self, "err", "")}
        import statistics
        names = [n for b, n in self.REASONS.items() if self.reasons & b and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None, "sm_max_mhz": self.max_mhz,
                "reasons": names, "samples": len(self.samples), "samples_in_timed_region": len(self.timed_samples),
                "sm_mhz_in_timed_region": statistics.median(self.timed_samples) if self.timed_samples else None}


# ---------------------------------------------------------------------------
# the oracle on the host cores (CPU baseline and the reference arm)
# ---------------------------------------------------------------------------
def oracle_sample_steps(n_steps: int, n_layers: int, want: int = 4) -> list[int]:
    """Steps of layer 0 (step s runs layer s mod n_layers) that the workload holds,
    at most `want` of them and never none: the oracle baseline runs layer 0's
    factors on those steps' tokens and routing."""
    n_layers = max(1, n_layers)
    steps = list(range(0, max(1, n_steps), n_layers))[:max(1, want)]
    return steps or [0]


class OracleSample:
    """Pre-packed oracle inputs for a few layer steps (packing untimed).

    factors: {"gate"|"up": {"phi_t", "amps", "comps", "widths"}} as torch tensors
    (any device; only the routed experts are copied to the host); steps: a list
    of (x [T][d_in] fp16, ids [T][top_k] int32, gate_w [T][top_k] f32) tensors.
    Uses synth's tensors and the oracle only: no part of the CUDA library."""

    def __init__(self, factors: dict, steps: list, rank: int, frac: float = 1.0):
        import numpy as np
        import torch
        import oracle
        oracle.build()
        self.o = oracle
        self.r_sub = max(1, int(round(frac * rank)))
        self.frac = self.r_sub / rank
        self.items = []
        for x_t, ids_t, g_t in steps:
            ids = ids_t.cpu().numpy()
            g = g_t.cpu().numpy()
            x = x_t.cpu().numpy().view(np.uint16)
            ex = sorted(set(int(v) for v in ids.ravel()))
            remap = np.vectorize({e: j for j, e in enumerate(ex)}.get)(ids).astype(np.int32)
            per = {}
            for name in ("gate", "up"):
                h = factors[name]
                sel = torch.as_tensor(ex, device=h["comps"].device)
                comps = h["comps"][sel][:, :self.r_sub].cpu().numpy()
                w = h["widths"][sel][:, :self.r_sub].cpu().numpy()
                a = h["amps"][sel][:, :self.r_sub].cpu().numpy()
                sc, _ = oracle.compute_scales(comps, w)
                blob, _ = oracle.pack(comps, w, sc, a)
                phi = h["phi_t"][:self.r_sub].cpu().numpy().view(np.uint16)
                per[name] = (blob, phi)
            self.items.append((x, remap, g, per))

    def run(self, i: int):
        x, ids, g, per = self.items[i % len(self.items)]
        for name in ("gate", "up"):
            blob, phi = per[name]
            Z = self.o.shared_proj(phi, x)
            self.o.expert_forward(blob, Z, ids, g, want_experts=False)


def time_oracle(sample: OracleSample, steps: int | None, seconds: float | None) -> tuple[float, int]:
    n, t0 = 0, time.perf_counter()
    while True:
        sample.run(n)
        n += 1
        el = time.perf_counter() - t0
        if steps is not None and n >= steps:
            break
        if seconds is not None and el >= seconds:
            break
    return el, n


def cores_used() -> int:
    return 1  # the oracle is single-threaded C


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def time_oracle_threads(sample, threads: int, seconds: float) -> tuple[float, int]:
    """The oracle on `threads` host threads at once, each running whole layer steps
    (its C calls release the interpreter lock; it keeps no mutable global state):
    elapsed seconds and steps completed."""
    import threading
    counts = [0] * threads
    deadline = time.perf_counter() + seconds

    def work(k):
        i = k
        while time.perf_counter() < deadline:
            sample.run(i)
            counts[k] += 1
            i += threads

    ts = [threading.Thread(target=work, args=(k,)) for k in range(threads)]
    t0 = time.perf_counter()
    for t in ts:
        t.start()
    for t in ts:
        t.join()
    return time.perf_counter() - t0, sum(counts)


# ---------------------------------------------------------------------------
# arms
# ---------------------------------------------------------------------------
def load_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# DRAM traffic of the dominant kernel comes from a committed ncu summary, which
# records the SHA-256 of the sources it was taken on; once those change the
# figure no longer describes the kernel and is reported as null.
TRAFFIC_SUMMARY = os.path.join(ROOT, "profiles", "k_layer_t1_qwen_t1.md")
TRAFFIC_SOURCES = ("mixed_precision_decode_b200/csrc/layer_t1.cu", "mixed_precision_decode_b200/csrc/common.cuh")


def sources_sha256(paths=TRAFFIC_SOURCES) -> str:
    import hashlib
    h = hashlib.sha256()
    for rel in paths:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def measured_traffic(config_name: str):
    """dram__bytes_read.sum + dram__bytes_write.sum per launch, or None."""
    if config_name != "qwen_t1":
        return None
    try:
        kv = {}
        with open(TRAFFIC_SUMMARY) as f:
            for line in f:
                if line.startswith("- `") and "`: " in line:
                    k, v = line[3:].split("`: ", 1)
                    kv[k.strip()] = v.strip().strip("`")
        if kv.get("sources_sha256") != sources_sha256():
            return None
        return float(kv["dram_bytes_per_launch"])
    except (OSError, KeyError, ValueError):
        return None


def workload_config(cfg, T, n_layers):
    """The workload's description, the same for both arms (nothing measured in it)."""
    return {"workload": f"{cfg.name}: spectral MoE gate/up layer, Qwen3-30B-A3B-shaped" if cfg.name.startswith("qwen")
            else cfg.name,
            "d_in": cfg.d_in, "d_out": cfg.d_out, "experts": cfg.n_experts, "top_k": cfg.top_k, "rank": cfg.rank,
            "tokens_per_step": T, "widths": "8:2% 4:8% 3:20% 2:40% 1:20% 0:10% (~2.08 bits)"
            if cfg.name in ("qwen_t1", "qwen_stack") else str(cfg.width_fracs),
            "l2": f"inputs larger than L2: {n_layers} distinct seeded layer copies rotated, each step its own "
                  f"token and routing",
            "routing": cfg.routing}


def weak_scaling_throughput(world: int, steps: int, tokens: int, ms_max: float):
    """Whole-job tokens/s and seconds per step: every rank runs `steps` steps of
    `tokens` tokens on its own replica; the job takes the slowest rank's time."""
    sec = ms_max / 1e3
    return world * steps * tokens / sec, sec / steps


def run_ours(args, dist):
    import numpy as np
    import torch
    from mixed_precision_decode_b200 import synth

    cfg = synth.CONFIGS[args.config]
    if args.tokens:
        cfg = synth.scaled(cfg, tokens=args.tokens)
    T = cfg.tokens
    K, W = args.steps, args.warmup
    G = max(1, min(K, args.graph_steps))
    L = args.layers
    n_steps_data = max(G, L)
    want_cpu = dist.rank == 0 and dist.world == 1 and not args.no_cpu_baseline
    wl = Workload(cfg, args.layers, n_steps_data, seed_base=10_000 + 1000 * dist.rank, keep_comps_of_layer0=want_cpu)
    stream = torch.cuda.current_stream()

    # algorithmic bytes per step, averaged over the K timed steps (step s: layer s mod L, data s mod n)
    pairs = {}
    for s in range(K):
        key = (wl.layer_of(s), wl.data_of(s))
        pairs[key] = pairs.get(key, 0) + 1
    bys = {key: algorithmic_bytes(cfg, wl.counts[key[0]], wl.ids[key[1]].cpu().numpy(), T) for key in pairs}
    alg = {k: float(sum(bys[key][k] * n for key, n in pairs.items()) / K) for k in next(iter(bys.values()))}
    # shared-memory wavefronts of the multi-token expert lookups per step (T > 1)
    lds_wf = float(sum(lds_wavefronts(cfg, wl.counts[key[0]], wl.ids[key[1]].cpu().numpy(), T) * n
                       for key, n in pairs.items()) / K) if T > 1 else 0.0

    # Steps run as a decode loop over a continuing rotation: timed step s (0..K-1)
    # is layer s mod L, and the K steps are captured in graphs of up to G steps
    # that continue the rotation.  Before them, an untimed graph of one whole
    # rotation (steps -L..-1) ends on layer L-1, so the first timed step's layer
    # was last read L steps earlier (L x the step's bytes, several times L2).
    # Each call names the step that runs next (the chained loop prefetches it).
    side = torch.cuda.Stream()

    def capture_range(start, n, chained):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=side):
            for s in range(start, start + n):
                wl.step(s, next_s=(s + 1) if chained else None)
        return g

    def capture(chained):
        for s in range(-W - L, -L):  # eager warm-up, W steps
            wl.step(s, next_s=(s + 1) if chained else None)
        torch.cuda.synchronize()
        pre = capture_range(-L, L, chained)
        gs = [capture_range(i, min(G, K - i), chained) for i in range(0, K, G)]
        pre.replay()
        for g in gs[:2]:
            g.replay()
        torch.cuda.synchronize()
        return pre, gs

    def preload_replays(pre, seconds):
        """Replays of the one-rotation graph that keep the GPU under this same load
        for about `seconds` (untimed; clocks are sampled meanwhile)."""
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(3):
            pre.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        t = max(1e-6, e0.elapsed_time(e1) / 3e3)
        return int(min(5000, max(2, math.ceil(seconds / t))))

    def timed(pre, gs, clocks=None, nvtx=False, n_pre=0):
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        dist.barrier()
        torch.cuda.synchronize()
        if clocks:
            clocks.timed_events = (ev0, ev1)
            clocks.__enter__()
        for _ in range(n_pre):  # untimed: the same steps, so the clocks are read under this load
            pre.replay()
        if clocks:
            clocks.sample_now()
        if nvtx:
            torch.cuda.nvtx.range_push("timed")
        ev0.record(stream)
        for g in gs:
            g.replay()
        ev1.record(stream)
        if clocks:
            clocks.sample_now()
        torch.cuda.synchronize()
        if nvtx:
            torch.cuda.nvtx.range_pop()
        if clocks:
            clocks.__exit__(None, None, None)
        dist.barrier()
        return dist.max(ev0.elapsed_time(ev1))

    # the same loop as a chained decode loop (next layer's Phi^T prefetched into L2), reported beside
    ms_chained = None
    if not args.no_chained:
        pre, graphs = capture(True)
        ms_chained = timed(pre, graphs, n_pre=1)
        del pre, graphs
    pre, graphs = capture(False)
    n_pre = preload_replays(pre, args.clock_window)
    clocks = ClockSampler(torch.cuda.current_device(), period_s=0.0)
    ms = timed(pre, graphs, clocks, nvtx=True, n_pre=n_pre)
    del pre, graphs
    value, step_s = weak_scaling_throughput(dist.world, K, T, ms)

    peak, peak_kind = load_peak()
    achieved = alg["total"] / step_s / 1e9
    launches_per_step = kernels_per_step(wl)

    # end to end through the public API: pinned host inputs -> device, forward, outputs -> pinned host
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(wl, cfg, T, min(K, 2000), dist)

    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": dist.world, "steps": K, "warmup": W,
        "ms_per_step": step_s * 1e3, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32", "data": "synthetic (seeded random factors of the layer's shape; no checkpoint)",
        "config": workload_config(cfg, T, args.layers),
        "workload_bytes": {"resident_gb": wl.blob_bytes_total() / 1e9, "mb_per_step": alg["total"] / 1e6,
                           "distinct_experts_per_step": alg["distinct_experts"]},
        "roofline": {"bound": "hbm", "kernel": dominant_kernel(launches_per_step), "achieved": achieved, "peak": peak,
                     "peak_kind": peak_kind, "unit": "GB/s", "frac": achieved / peak,
                     "traffic": measured_traffic(cfg.name) if launches_per_step == 1 and T == 1 else None,
                     "algorithmic_bytes_per_launch": alg["total"], "bytes_breakdown": {k: alg[k] for k in
                                                                                       ("phi", "planes", "meta", "act")},
                     "duration_us": step_s * 1e6},
        "gpu_launches": launches_per_step * K,
        "clocks": dict(clocks.summary(), window=f"sampled over {n_pre} untimed replays of one rotation ({n_pre * L} "
                                                    f"steps of the same loop) and the timed region right after them"),
        "e2e": e2e,
    }
    if T > 1:
        # the expert lookups' own bound: shared-memory wavefronts over the whole step's time
        # (a lower bound on the kernel's rate), against 128 B per clock per SM at the sampled clock
        lds_peak = lds_peak_gbs(line["clocks"].get("sm_mhz") or 1965.0, torch.cuda.get_device_properties(0).multi_processor_count)
        lds_achieved = lds_wf * 128 / step_s / 1e9
        line["roofline_lds"] = {"bound": "lds", "kernel": "k_expert_mt (table lookups, both projections)",
                                "achieved": lds_achieved, "peak": lds_peak, "peak_kind": "unit counts x sampled SM clock",
                                "unit": "GB/s", "frac": lds_achieved / lds_peak,
                                "wavefronts_per_step": lds_wf, "duration_us": step_s * 1e6}
    if ms_chained is not None:
        value_ch, step_ch = weak_scaling_throughput(dist.world, K, T, ms_chained)
        line["chained"] = {"value": value_ch, "ms_per_step": step_ch * 1e3,
                           "roofline_frac": alg["total"] / step_ch / 1e9 / peak,
                           "how": "the same graph-replayed loop through bitsmoe_layer_forward_chained: each call "
                                  "prefetches the next step's layer Phi^T into L2 while it evaluates experts"}
    if want_cpu:
        steps = [(wl.x[d], wl.ids[d], wl.gw[d]) for d in oracle_sample_steps(wl.n_steps, L)]
        samp = OracleSample(wl.host0, steps, cfg.rank)
        el, n = time_oracle(samp, None, args.cpu_seconds)
        line["cpu_baseline"] = {"value": n * T / el, "unit": "tokens/s", "cores": cores_used(), "kind": "oracle",
                                "sample": f"{n} full layer steps ({len(samp.items)} distinct pre-packed steps of "
                                          f"layer 0, packing untimed), {el:.1f} s, single-threaded C oracle"}
        # the same oracle on every host core: independent layer steps on one thread per core
        nthr = host_cores()
        el_a, n_a = time_oracle_threads(samp, nthr, args.cpu_seconds)
        line["cpu_baseline"]["all_cores"] = {
            "value": n_a * T / el_a, "unit": "tokens/s", "cores": nthr, "cpu": cpu_model(),
            "sample": f"{n_a} full layer steps on {nthr} threads (one per core, each its own steps), {el_a:.1f} s"}
    if dist.rank == 0:
        print(json.dumps(line), flush=True)


def down_bytes(cfg, ids_step, T) -> dict:
    """Bytes the down step must move for one layer step: the dense fp16 down matrix
    [d_in][d_out] of each distinct routed expert, the gate and up expert outputs
    (fp32, T x top_k x d_out each), the routing and the fp32 output."""
    import numpy as np
    experts = np.unique(ids_step.reshape(-1))
    w = int(len(experts)) * cfg.d_in * cfg.d_out * 2
    act = 2 * T * cfg.top_k * cfg.d_out * 4 + T * cfg.top_k * 8 + T * cfg.d_in * 4
    return {"w_down": w, "act": act, "total": w + act}


def run_ffn(args, dist):
    """The whole expert FFN as a decode loop: per step one bitsmoe_ffn_forward call --
    the spectral gate/up layer (Y_experts of both projections), then SiLU(gate) * up,
    the dense fp16 down projection and the slot-order routed sum.  The step loop and,
    separately, a loop of bitsmoe_ffn_down calls alone (the down kernel's own
    roofline) are graph-replayed over L layer copies."""
    import torch
    from mixed_precision_decode_b200 import bitsmoe as B
    from mixed_precision_decode_b200 import synth
    from mixed_precision_decode_b200.layer import SpectralMoEFFN

    cfg = synth.CONFIGS[args.config]
    if args.tokens:
        cfg = synth.scaled(cfg, tokens=args.tokens)
    T = cfg.tokens
    K, W = args.steps, args.warmup
    G = max(1, min(K, args.graph_steps))
    L = args.layers
    dev = torch.device("cuda")
    wl = Workload(cfg, L, max(G, L), seed_base=10_000 + 1000 * dist.rank)
    ffns = [SpectralMoEFFN(layer, synth.make_down(cfg, synth.make_generator(20_000 + 1000 * dist.rank + l, dev), dev))
            for l, layer in enumerate(wl.layers)]
    bufs = [layer.forward(wl.x[0], wl.ids[0], wl.gw[0], want_experts=True) for layer in wl.layers]
    outs = [torch.empty((T, cfg.d_in), dtype=torch.float32, device=dev) for _ in range(L)]
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    side = torch.cuda.Stream()

    n_dws = B.ffn_down_workspace_bytes(ffns[0].dims, T)
    down_ws = torch.empty(max(n_dws, 256), dtype=torch.uint8, device=dev)

    def down_step(s):
        l, d = wl.layer_of(s), wl.data_of(s)
        f = ffns[l]
        B.ffn_down(f.dims, f.w_down, bufs[l]["Y_experts_gate"], bufs[l]["Y_experts_up"], wl.ids[d], wl.gw[d], T,
                   outs[l], down_ws, n_dws)

    def ffn_step(s):
        l, d = wl.layer_of(s), wl.data_of(s)
        if args.ffn_two_calls:
            wl.layers[l].forward(wl.x[d], wl.ids[d], wl.gw[d], out=bufs[l], want_experts=True)
            down_step(s)
        else:
            ffns[l].forward(wl.x[d], wl.ids[d], wl.gw[d], out=outs[l], gate_up=bufs[l])

    def graphs_of(fn):
        for s in range(-W - L, -L):
            fn(s)
        torch.cuda.synchronize()
        def cap(start, n):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=side):
                for s in range(start, start + n):
                    fn(s)
            return g
        pre = cap(-L, L)
        gs = [cap(i, min(G, K - i)) for i in range(0, K, G)]
        pre.replay()
        torch.cuda.synchronize()
        return pre, gs

    def timed(pre, gs, clocks=None, n_pre=1, nvtx=None):
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        dist.barrier()
        torch.cuda.synchronize()
        if clocks:
            clocks.timed_events = (ev0, ev1)
            clocks.__enter__()
        for _ in range(n_pre):
            pre.replay()
        if clocks:
            clocks.sample_now()
        if nvtx:
            torch.cuda.nvtx.range_push(nvtx)
        ev0.record(stream)
        for g in gs:
            g.replay()
        ev1.record(stream)
        if clocks:
            clocks.sample_now()
        torch.cuda.synchronize()
        if nvtx:
            torch.cuda.nvtx.range_pop()
        if clocks:
            clocks.__exit__(None, None, None)
        dist.barrier()
        return dist.max(ev0.elapsed_time(ev1))

    pre, gs = graphs_of(down_step)
    ms_down = timed(pre, gs, n_pre=2, nvtx="timed_down")
    del pre, gs
    pre, gs = graphs_of(ffn_step)
    clocks = ClockSampler(torch.cuda.current_device(), period_s=0.0)
    ms = timed(pre, gs, clocks, n_pre=max(2, int(args.clock_window * 1e3 / max(1e-3, L * 0.02))), nvtx="timed")
    del pre, gs
    value, step_s = weak_scaling_throughput(dist.world, K, T, ms)
    down_s = ms_down / 1e3 / K

    counts = {}
    for s in range(K):
        key = (wl.layer_of(s), wl.data_of(s))
        counts[key] = counts.get(key, 0) + 1
    db = {k: sum(down_bytes(cfg, wl.ids[key[1]].cpu().numpy(), T)[k] * n for key, n in counts.items()) / K
          for k in ("w_down", "act", "total")}
    gb = sum(algorithmic_bytes(cfg, wl.counts[key[0]], wl.ids[key[1]].cpu().numpy(), T)["total"] * n
             for key, n in counts.items()) / K
    peak, peak_kind = load_peak()
    n_down = B.ffn_down_launches(ffns[0].dims, T)
    ach = db["total"] / down_s / 1e9
    line = {
        "metric": "decode tokens/s, expert FFN: spectral gate/up + SiLU(gate)*up + dense fp16 down projection",
        "value": value, "unit": "tokens/s", "n_gpus": dist.world, "steps": K, "warmup": W,
        "ms_per_step": step_s * 1e3, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32", "data": "synthetic (seeded random factors and down weights of the layer's shape)",
        "config": dict(workload_config(cfg, T, L), down="dense fp16 [E][d_in][d_out] per expert, N(0,1)/sqrt(d_out)"),
        "roofline": {"bound": "hbm", "kernel": "k_down_t1" if n_down == 1 else
                     f"k_route + {'k_down_tc' if cfg.d_out <= 2048 else 'k_down_mt'} + k_combine",
                     "achieved": ach, "peak": peak, "peak_kind": peak_kind, "unit": "GB/s", "frac": ach / peak,
                     "traffic": None, "algorithmic_bytes_per_launch": db["total"] if n_down == 1 else None,
                     "algorithmic_bytes_per_step": db["total"], "duration_us": down_s * 1e6,
                     "how": "the down calls alone, graph-replayed over the layer copies, timed with CUDA events"},
        "step_roofline": {"achieved": (gb + db["total"]) / step_s / 1e9, "peak": peak,
                          "frac": (gb + db["total"]) / step_s / 1e9 / peak,
                          "bytes_per_step": {"gate_up": gb, "down": db["total"]}},
        "gpu_launches": (B.layer_launches(wl.layers[0].gate.plan, wl.layers[0].up.plan, T) + n_down
                         if args.ffn_two_calls else ffns[0].launches(T)) * K,
        "ffn_call": "bitsmoe_layer_forward + bitsmoe_ffn_down" if args.ffn_two_calls else "bitsmoe_ffn_forward",
        "clocks": dict(clocks.summary(), window="untimed replays of one rotation and the timed region"),
    }
    if dist.rank == 0:
        print(json.dumps(line), flush=True)


def fp32_peak_tflops(sm_mhz: float, sms: int = 148) -> float:
    """fp32 FMA throughput from the unit counts: 128 lanes per SM, 2 flops per FMA."""
    return 128 * 2 * sms * sm_mhz * 1e6 / 1e12


def run_ssd(args, dist):
    """The offline step for one projection of the configuration's shape, as
    layer.decompose_and_pack runs it: the shared-basis decomposition of seeded
    synthetic expert matrices W_e ~ N(0, 1/d_in) (fp32), the widths of the
    configuration's allocation by descending amplitude (host), quantisation and
    packing.  Each repetition is timed with CUDA events per stage."""
    import torch
    from mixed_precision_decode_b200 import bitsmoe as B
    from mixed_precision_decode_b200 import synth
    from mixed_precision_decode_b200.layer import PackedProjection

    cfg = synth.CONFIGS[args.config]
    E, d_out, d_in, r = cfg.n_experts, cfg.d_out, cfg.d_in, cfg.rank
    dev = torch.device("cuda")
    gen = synth.make_generator(30_000 + 1000 * dist.rank, dev)
    W = (torch.randn((E, d_out, d_in), generator=gen, device=dev) * d_in ** -0.5).contiguous()
    counts = synth.width_counts(cfg)
    order, cnt = [b for b, _ in counts], [n for _, n in counts]
    n_ws = B.ssd_workspace_bytes(E, d_out, d_in, r)
    ws = torch.empty(n_ws, dtype=torch.uint8, device=dev)
    phi_t = torch.empty((r, d_in), dtype=torch.float16, device=dev)
    amps = torch.empty((E, r), dtype=torch.float32, device=dev)
    comps = torch.empty((E, r, d_out), dtype=torch.float32, device=dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream()

    if args.fqcm:
        from mixed_precision_decode_b200.layer import fqcm_widths
        xc = torch.randn((args.calib_tokens, d_in), generator=gen, device=dev).to(torch.float16)
        ids_c, gw_c = synth.make_routing(cfg, gen, dev, args.calib_tokens)
        avg_bits = sum(b * n for b, n in counts) / r

    def once(timing):
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        ev[0].record(stream)
        B.ssd_decompose(W, r, phi_t, amps, comps, ws, n_ws, status=st)
        ev[1].record(stream)
        torch.cuda.synchronize()  # the stages run one after another
        t0 = time.perf_counter()
        if args.fqcm:  # z of the calibration tokens on the GPU, then beta, eps and the allocation on the host
            widths, _, _ = fqcm_widths({"phi_t": phi_t, "amps": amps, "comps": comps}, xc, ids_c, gw_c, avg_bits)
        else:
            widths = torch.from_numpy(B.assign_widths(amps.cpu().numpy(), order, cnt))  # D2H of a, host sort
        t_w = time.perf_counter() - t0
        ev_p0 = torch.cuda.Event(enable_timing=True)
        ev_p0.record(stream)
        pk = PackedProjection.from_factors(phi_t, amps, comps, widths, cfg.top_k, status=st)
        ev[2].record(stream)
        torch.cuda.synchronize()
        if timing is not None:
            timing["decompose"].append(ev[0].elapsed_time(ev[1]))
            timing["widths"].append(t_w * 1e3)
            timing["pack"].append(ev_p0.elapsed_time(ev[2]))
        return pk

    for _ in range(max(1, args.warmup)):
        once(None)
    timing = {"decompose": [], "widths": [], "pack": []}
    dist.barrier()
    for _ in range(args.steps):
        pk = once(timing)
    dist.barrier()
    assert B.read_status(st) == 0
    med = {k: sorted(v)[len(v) // 2] for k, v in timing.items()}
    total = med["decompose"] + med["widths"] + med["pack"]
    total_max = dist.max(total)
    flops = 2 * 2 * (E * d_out) * d_in * r  # W_cat^T W_cat and W_cat Phi
    peak = fp32_peak_tflops(1965.0)
    ach = flops / (med["decompose"] * 1e-3) / 1e12
    line = {"metric": "offline decomposition + widths + packing time per projection", "value": total_max,
            "unit": "ms", "n_gpus": dist.world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": total_max, "higher_is_better": False, "scaling": "weak", "vs_baseline": None,
            "dtype": "f32", "data": "synthetic expert matrices N(0, 1/d_in), seeded",
            "config": {"workload": f"{cfg.name}: one projection, {E} experts of {d_out} x {d_in}, rank {r}",
                       "widths": (f"FQCM allocation at {sum(b * n for b, n in counts) / r:.4f} average bits, "
                                  f"{args.calib_tokens} seeded calibration tokens") if args.fqcm else str(counts)},
            "stages_ms": med,
            "roofline": {"bound": "alu", "kernel": "decomposition (two fp32 GEMMs in cuBLAS, fp32 eigensolver)",
                         "achieved": ach, "peak": peak, "unit": "TFLOP/s", "frac": ach / peak,
                         "peak_kind": "fp32 FMA units x clocks.max.sm (1965 MHz)",
                         "flops_per_step": flops, "duration_us": med["decompose"] * 1e3},
            "blob_bytes": pk.plan.blob_bytes}
    if dist.rank == 0:
        print(json.dumps(line), flush=True)


def kernels_per_step(wl) -> int:
    from mixed_precision_decode_b200 import bitsmoe as B
    L = wl.layers[0]
    return B.layer_launches(L.gate.plan, L.up.plan, wl.cfg.tokens)


def dominant_kernel(n_launches: int) -> str:
    return "k_layer_t1 (fused single-token layer)" if n_launches == 1 else \
        "whole step: k_route, shared projection x2 (k_proj_tc or k_shared_proj), k_expert_mt x2, k_combine x2"


def run_e2e(wl, cfg, T, n, dist):
    """The public API as a decode loop calls it, one step after another: the step's
    inputs (x, routing ids, gate weights) are packed in one pinned host buffer and
    copied to the device in one transfer, the layer forward runs on views of that
    buffer, and both routed sums (one [2][T][d_out] buffer) come back in one
    transfer."""
    import torch
    m = wl.n_steps
    xb, ib, gb = T * cfg.d_in * 2, T * cfg.top_k * 4, T * cfg.top_k * 4
    o_i = (xb + 15) // 16 * 16
    o_g = o_i + (ib + 15) // 16 * 16
    nbytes = o_g + gb
    host_in = torch.empty((m, nbytes), dtype=torch.uint8).pin_memory()
    for s in range(m):
        host_in[s, :xb] = wl.x[s].cpu().contiguous().view(torch.uint8).reshape(-1)
        host_in[s, o_i:o_i + ib] = wl.ids[s].cpu().contiguous().view(torch.uint8).reshape(-1)
        host_in[s, o_g:o_g + gb] = wl.gw[s].cpu().contiguous().view(torch.uint8).reshape(-1)
    dev_in = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    xd = dev_in[:xb].view(torch.float16).view(T, cfg.d_in)
    idd = dev_in[o_i:o_i + ib].view(torch.int32).view(T, cfg.top_k)
    gwd = dev_in[o_g:o_g + gb].view(torch.float32).view(T, cfg.top_k)
    dev_out = torch.empty((2, T, cfg.d_out), dtype=torch.float32, device="cuda")
    out = {"Y_sum_gate": dev_out[0], "Y_sum_up": dev_out[1]}
    host_out = torch.empty((m, 2, T, cfg.d_out), dtype=torch.float32).pin_memory()
    stream = torch.cuda.current_stream()

    def one(s):
        s = s % m
        dev_in.copy_(host_in[s], non_blocking=True)
        wl.layers[wl.layer_of(s)].forward(xd, idd, gwd, out=out)
        host_out[s].copy_(dev_out, non_blocking=True)

    for s in range(min(n, 50)):
        one(s)
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dist.barrier()
    torch.cuda.synchronize()
    ev0.record(stream)
    for s in range(n):
        one(s)
    ev1.record(stream)
    torch.cuda.synchronize()
    dist.barrier()
    sec = dist.max(ev0.elapsed_time(ev1)) / 1e3

    # The same steps captured in CUDA graphs: each step's H2D copy (from its own pinned
    # slot), the layer call and the D2H copy are graph nodes, so the host enqueues
    # nothing per step; the copies still cross PCIe every step.
    side = torch.cuda.Stream()
    G = min(n, 500)
    graphs = []
    for start in range(0, n, G):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=side):
            for s in range(start, min(n, start + G)):
                one(s)
        graphs.append(g)
    graphs[0].replay()
    torch.cuda.synchronize()
    dist.barrier()
    torch.cuda.synchronize()
    ev0.record(stream)
    for g in graphs:
        g.replay()
    ev1.record(stream)
    torch.cuda.synchronize()
    dist.barrier()
    sec_g = dist.max(ev0.elapsed_time(ev1)) / 1e3
    del graphs
    return {"value": dist.world * n * T / sec, "unit": "tokens/s", "h2d_bytes_per_step": nbytes,
            "d2h_bytes_per_step": 2 * T * cfg.d_out * 4, "steps": n,
            "how": "eager public-API loop, steps serialised: one pinned H2D of the step's packed x/ids/gate_w, "
                   "SpectralMoELayer.forward on views of it, one D2H of both Y_sum; CUDA events on the stream",
            "graph": {"value": dist.world * n * T / sec_g, "unit": "tokens/s", "us_per_step": sec_g / n * 1e6,
                      "how": "the same steps (H2D copy, layer call, D2H copy each) captured in CUDA graphs "
                             f"of up to {G} steps and replayed"}}


def host_workload(cfg, seed: int, n_steps: int) -> tuple[dict, list]:
    """Layer-0-style factors of both projections and n_steps (x, ids, gate_w),
    drawn by synth on the CPU: the same shapes and distributions as the GPU
    workload, from CPU generators (so not the same values).  No part of the
    CUDA library is used."""
    import torch
    from mixed_precision_decode_b200 import synth
    cpu = torch.device("cpu")
    gen = synth.make_generator(seed, cpu)
    factors = {name: synth.make_projection(cfg, gen, cpu) for name in ("gate", "up")}
    gen = synth.make_generator(seed + 999_983, cpu)
    steps = []
    for _ in range(n_steps):
        x = torch.randn((cfg.tokens, cfg.d_in), generator=gen).to(torch.float16)
        ids, gw = synth.make_routing(cfg, gen, cpu, cfg.tokens)
        steps.append((x, ids, gw))
    return factors, steps


def run_reference(args, dist):
    """The oracle (plain single-threaded C, fp64) on the host cores, timed per
    step on a bounded sample of the same workload.  Rank 0 only; the inputs come
    from synth and the oracle alone (the CUDA library is never loaded)."""
    from mixed_precision_decode_b200 import synth

    if dist.rank != 0:
        return
    cfg = synth.CONFIGS[args.config]
    if args.tokens:
        cfg = synth.scaled(cfg, tokens=args.tokens)
    T = cfg.tokens
    K, W = args.steps, args.warmup
    factors, steps = host_workload(cfg, 10_000, 4)
    probe = OracleSample(factors, steps[:1], cfg.rank, 1.0)
    t0 = time.perf_counter()
    probe.run(0)
    t_full = time.perf_counter() - t0
    budget = 150.0  # seconds of timed oracle work for the whole run
    frac = min(1.0, budget / max(1e-9, (K + W) * t_full))
    samp = OracleSample(factors, steps, cfg.rank, frac)
    del factors
    for i in range(W):
        samp.run(i)
    el, n = time_oracle(samp, K, None)
    value = samp.frac * n * T / el
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": dist.world, "steps": K,
        "warmup": W, "ms_per_step": el / n * 1e3 / samp.frac, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded random factors of the layer's shape)",
        "config": workload_config(cfg, T, args.layers),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores_used(), "kind": "oracle",
                         "cpu": cpu_model(),
                         "sample": f"each step: {samp.r_sub} of {cfg.rank} spectral components (fraction "
                                   f"{samp.frac:.4f}) of a full layer step, both projections; value scaled by "
                                   f"1/fraction; 4 distinct pre-packed steps drawn on the CPU (packing untimed)"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    dist = Dist(args.gpus)
    try:
        if args.impl == "reference":
            run_reference(args, dist)
        elif args.ffn:
            run_ffn(args, dist)
        elif args.ssd:
            run_ssd(args, dist)
        else:
            run_ours(args, dist)
    finally:
        dist.close()


if __name__ == "__main__":
    main()
