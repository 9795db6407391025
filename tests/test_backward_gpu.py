"""Backward pass through the C ABI against the fp64 oracle's gradients of the
definition (oracle.attention_grad, pinned by finite differences).  Needs a
B200."""
import json
import os

import numpy as np
import pytest
import torch

import oracle
import linear_cost_attention_b200 as sata
from sata_inputs import make_qkv
from tests.parity import TOL

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from linear_cost_attention_b200 import build

    build.build()
    torch.cuda.set_device(0)
    yield
    assert sata.sata_get_error() == sata.SATA_OK


def grad_err(got, ref):
    """Largest |difference| over the largest |reference| entry, per head."""
    got = np.asarray(got, dtype=np.float64)
    d = np.max(np.abs(got - ref), axis=(-2, -1))
    return float(np.max(d / np.max(np.abs(ref), axis=(-2, -1))))


@pytest.mark.parametrize("B,H,N,dK,dV,P,dt", [
    (1, 1, 1, 8, 8, 4, "f32"),          # a single token
    (1, 2, 77, 16, 8, 4, "f32"),        # ragged tile, dK != dV
    (2, 2, 200, 32, 32, 4, "f32"),
    (1, 2, 300, 64, 64, 4, "bf16"),
    (1, 1, 130, 64, 64, 3, "f32"),
    (2, 1, 64, 8, 16, 1, "f32"),        # P = 1: dq = dk = 0
    (1, 2, 96, 16, 16, 5, "bf16"),
])
def test_backward_matches_oracle(B, H, N, dK, dV, P, dt):
    q, k, v = make_qkv(B, H, N, dK, dV, seed=N + 13 * dK + P, dtype=dt)
    g = torch.Generator().manual_seed(N + P)
    dout = torch.randn(B, H, N, dV, generator=g)
    dq, dk, dv = sata.attention_backward(q.cuda(), k.cuda(), v.cuda(), dout.cuda(), P)
    torch.cuda.synchronize()
    rq, rk, rv = oracle.attention_grad(q, k, v, dout, P)
    tol = TOL[dt]
    errs = {}
    # a gradient that is exactly zero (P = 1, or a single token whose output
    # is v_0 whatever q, k are) is compared on the scale of the largest one
    scale = max(float(np.max(np.abs(r))) for r in (rq, rk, rv))
    for name, got, ref in (("dq", dq, rq), ("dk", dk, rk), ("dv", dv, rv)):
        got = got.cpu().double().numpy()
        assert np.isfinite(got).all()
        if np.max(np.abs(ref)) == 0:
            errs[name] = float(np.max(np.abs(got))) / scale
            continue
        errs[name] = grad_err(got, ref)
    path = os.environ.get("SATA_PARITY_LOG")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps({"case": f"backward {B}x{H}x{N} dK={dK} dV={dV} P={P} {dt}",
                                **errs, "tol": tol}) + "\n")
    for name, e in errs.items():
        assert e <= tol, (name, e)
