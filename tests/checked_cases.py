"""Run by tests/test_gpu_checked.py in a process with BITSMOE_CHECKED=1: the small
parity cases through the bounds-checked library, at one token (the fused kernel)
and at every token (the multi-token kernels), checked against the oracle.  Any
index outside its buffer sets the status bit ST_BOUNDS; the status must stay 0.
Prints one line per case; exits non-zero on the first failure."""
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, HERE)
sys.path.insert(0, os.path.dirname(HERE))

import numpy as np  # noqa: E402
import torch  # noqa: E402

import oracle  # noqa: E402
from cases import SMALL, TOL, Case, oracle_tokens, rel_err, x_bits  # noqa: E402
from mixed_precision_decode_b200 import bitsmoe as B  # noqa: E402


def run_case(name, orc):
    case = Case(SMALL[name])
    assert B.read_status(case.status) == 0, f"{name}: packing status"
    T = case.cfg.tokens
    for toks in ([0], list(range(T))):
        sl = slice(toks[0], toks[-1] + 1)
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        out = case.layer.forward(case.x[sl].contiguous(), case.ids[sl].contiguous(), case.gate_w[sl].contiguous(),
                                 want_experts=True, want_z=True, status=st)
        s = B.read_status(st)
        assert s == 0, f"{name} T={len(toks)}: status {s}"
        for proj in ("gate", "up"):
            Zref = orc.shared_proj(case.host[proj]["phi_t"], x_bits(case)[sl])
            Ye_ref, Ys_ref = oracle_tokens(case, orc, proj, toks, Zref)
            assert rel_err(out[f"Y_experts_{proj}"].cpu().numpy(), Ye_ref) <= TOL, (name, proj, len(toks))
            assert rel_err(out[f"Y_sum_{proj}"].cpu().numpy(), Ys_ref) <= TOL, (name, proj, len(toks))
        print(f"ok {name} T={len(toks)} launches={B.layer_launches(case.proj['gate'].plan, case.proj['up'].plan, len(toks))}")


def main():
    assert B._LIB_PATH.endswith("libbitsmoe_checked.so"), B._LIB_PATH
    oracle.build()
    for name in ("tiny", "ragged", "one_expert"):
        run_case(name, oracle)
    print("checked ok")


if __name__ == "__main__":
    main()
