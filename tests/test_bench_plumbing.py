"""bench.py's host-side plumbing on CPU: which steps the oracle baseline samples
at the driver's arguments, and the reference arm end to end on a small config
(synth + oracle only: the CUDA library must not be loaded by that process)."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _n_steps_data(steps, graph_steps=1000, layers=16):
    # as run_ours sizes the pre-drawn steps
    return max(max(1, min(steps, graph_steps)), layers)


@pytest.mark.parametrize("steps,layers", [(20, 16), (1, 16), (20000, 16), (3, 1), (2, 2), (5, 7)])
def test_oracle_steps_exist_and_run_layer0(steps, layers):
    n = _n_steps_data(steps, layers=layers)
    got = bench.oracle_sample_steps(n, layers)
    assert 1 <= len(got) <= 4
    assert all(0 <= s < n for s in got)           # every sampled step is held by the workload
    assert all(s % layers == 0 for s in got)      # and runs layer 0, whose factors the oracle packs
    assert got == sorted(set(got))


def test_driver_arguments_sample_steps_0_and_16():
    # python bench.py --gpus 1 --steps 20 --warmup 5 (default --layers 16)
    assert bench.oracle_sample_steps(_n_steps_data(20), 16) == [0, 16]


def test_timed_steps_continue_the_rotation():
    # run_ours captures the K timed steps as graphs of G that continue the
    # rotation; step s runs layer s mod L on data s mod n
    class _W:
        n_steps, layers = 20, list(range(16))
        layer_of = bench.Workload.layer_of
        data_of = bench.Workload.data_of

    w = _W()
    K, G = 45, 20
    seq = [(w.layer_of(s), w.data_of(s)) for i in range(0, K, G) for s in range(i, min(i + G, K))]
    assert [l for l, _ in seq] == [s % 16 for s in range(K)]
    assert [d for _, d in seq] == [s % 20 for s in range(K)]
    # the preload rotation (-L .. -1) ends on layer L-1, right before layer 0
    assert [w.layer_of(s) for s in range(-16, 0)] == list(range(16))


def test_workload_config_is_measurement_free():
    from mixed_precision_decode_b200 import synth
    cfg = synth.CONFIGS["qwen_t1"]
    a = bench.workload_config(cfg, 1, 16)
    b = bench.workload_config(cfg, 1, 16)
    assert a == b and a["tokens_per_step"] == 1 and a["d_in"] == 2048


def test_reference_arm_uses_only_synth_and_oracle():
    code = (
        "import sys, json, io, contextlib; sys.path.insert(0, %r)\n"
        "sys.argv = ['bench.py', '--impl', 'reference', '--config', 'tiny', '--steps', '3', '--warmup', '1']\n"
        "import bench\n"
        "buf = io.StringIO()\n"
        "with contextlib.redirect_stdout(buf):\n"
        "    bench.main()\n"
        "maps = open('/proc/self/maps').read()\n"
        "print(json.dumps({'line': buf.getvalue().strip(), 'libbitsmoe': 'libbitsmoe.so' in maps}))\n" % ROOT)
    env = dict(os.environ)
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        env.pop(k, None)
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=300, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    out = json.loads(r.stdout.strip().splitlines()[-1])
    assert out["libbitsmoe"] is False
    line = json.loads(out["line"])
    assert line["impl"] == "reference" and line["steps"] == 3 and line["warmup"] == 1
    assert line["value"] > 0 and line["unit"] == "tokens/s" and line["higher_is_better"] is True
    assert line["config"] == bench.workload_config(__import__("mixed_precision_decode_b200.synth",
                                                                fromlist=["CONFIGS"]).CONFIGS["tiny"], 4, 16)
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0


def test_ffn_and_offline_byte_and_peak_formulas():
    """The FFN line's bytes: each distinct routed expert's fp16 down matrix once, plus
    the fp32 gate/up expert outputs, routing and output; the offline line's fp32
    peak from the unit counts."""
    import numpy as np
    from mixed_precision_decode_b200 import synth
    cfg = synth.CONFIGS["qwen_t1"]
    ids = np.array([[3, 7, 3, 9, 1, 2, 4, 5]])  # expert 3 twice: read once
    b = bench.down_bytes(cfg, ids, 1)
    assert b["w_down"] == 7 * 2048 * 768 * 2
    assert b["act"] == 2 * 1 * 8 * 768 * 4 + 1 * 8 * 8 + 1 * 2048 * 4
    assert b["total"] == b["w_down"] + b["act"]
    assert abs(bench.fp32_peak_tflops(1965.0) - 148 * 128 * 2 * 1.965e9 / 1e12) < 1e-9


def test_cli_modes_parse(monkeypatch):
    monkeypatch.setattr(sys, "argv", ["bench.py", "--ffn", "--ffn-two-calls", "--steps", "3"])
    a = bench.parse()
    assert a.ffn and a.ffn_two_calls and not a.ssd and a.steps == 3
    monkeypatch.setattr(sys, "argv", ["bench.py", "--ssd", "--fqcm", "--calib-tokens", "64"])
    a = bench.parse()
    assert a.ssd and a.fqcm and a.calib_tokens == 64 and not a.ffn
