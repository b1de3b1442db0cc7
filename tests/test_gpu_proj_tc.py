"""z = Phi^T X on the tensor cores (batches of 8+ tokens) against the oracle,
with ragged token counts, two token tiles and the Phi = I closed form."""
import numpy as np
import pytest
import torch

from cases import TOL, rel_err
from mixed_precision_decode_b200 import bitsmoe as B

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("T,d_in,r", [(8, 512, 128), (17, 512, 256), (64, 1024, 384), (300, 512, 128),
                                      (16, 2048, 2048)])
def test_proj_tc_against_oracle(orc, T, d_in, r):
    g = torch.Generator(device="cuda").manual_seed(T * 7 + r)
    phi_t = torch.randn((r, d_in), generator=g, device="cuda").to(torch.float16)
    x = torch.randn((T, d_in), generator=g, device="cuda").to(torch.float16)
    Z = torch.full((T, r), float("nan"), device="cuda")
    B.shared_proj(phi_t, x, Z, T, d_in, r)
    ref = orc.shared_proj(phi_t.cpu().numpy().view(np.uint16), x.cpu().numpy().view(np.uint16))
    assert rel_err(Z.cpu().numpy(), ref) <= TOL
    # the same products through the GEMV path agree closely (fp32 sums in another order)
    Z1 = torch.empty((1, r), device="cuda")
    B.shared_proj(phi_t, x[3:4].contiguous(), Z1, 1, d_in, r)
    assert rel_err(Z[3:4].cpu().numpy(), Z1.cpu().numpy()) <= 1e-5


def test_proj_tc_identity_is_exact():
    d = 512
    eye = torch.eye(d, dtype=torch.float16, device="cuda")
    x = torch.randn((24, d), device="cuda").to(torch.float16)
    Z = torch.empty((24, d), device="cuda")
    B.shared_proj(eye, x, Z, 24, d, d)
    assert torch.equal(Z, x.float())


def test_proj_tc_deterministic():
    g = torch.Generator(device="cuda").manual_seed(3)
    phi_t = torch.randn((256, 1024), generator=g, device="cuda").to(torch.float16)
    x = torch.randn((40, 1024), generator=g, device="cuda").to(torch.float16)
    a = torch.empty((40, 256), device="cuda")
    b = torch.empty((40, 256), device="cuda")
    B.shared_proj(phi_t, x, a, 40, 1024, 256)
    B.shared_proj(phi_t, x, b, 40, 1024, 256)
    assert torch.equal(a, b)
