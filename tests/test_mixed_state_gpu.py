"""The mixed-precision decode state (rows of degree <= 2 in fp32, the rest in
fp16) against the fp64 oracle, through the C ABI.  Needs a B200."""
import json
import os

import numpy as np
import pytest
import torch

import oracle
import linear_cost_attention_b200 as sata
from sata_inputs import WORKLOADS, DecodeStream, make_qkv, workload_inputs
from tests.parity import TOL, state_col_error

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from linear_cost_attention_b200 import build

    build.build()
    torch.cuda.set_device(0)
    yield
    assert sata.sata_get_error() == sata.SATA_OK


def record(name, **kw):
    path = os.environ.get("SATA_PARITY_LOG")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps({"case": name, **kw}) + "\n")


def row_err(got, ref):
    got = np.asarray(got, dtype=np.float64)
    return float(np.max(np.max(np.abs(got - ref), axis=-1) / np.max(np.abs(ref), axis=-1)))


@pytest.mark.parametrize("dK,P", [(8, 4), (64, 4), (16, 5), (32, 2)])
def test_fp32_rows_count(dK, P):
    import math

    assert sata.sata_state_fp32_rows(dK, P) == math.comb(dK + min(P, 3) - 1, min(P, 3) - 1)


def test_split_join_round_trip():
    B, H, dK, dV, P = 2, 3, 32, 32, 4
    m = sata.sata_basis_size(dK, P)
    g = torch.Generator().manual_seed(3)
    state = (torch.randn(B, H, m, dV + 1, generator=g) * 10).cuda()
    lo, hi = sata.split_state(state, P)
    m_lo = sata.sata_state_fp32_rows(dK, P)
    assert lo.shape == (B, H, m_lo, dV + 1) and hi.shape == (B, H, m - m_lo, dV + 1)
    torch.cuda.synchronize()
    assert torch.equal(lo, state[:, :, :m_lo])
    # fp16 rows: round to nearest, the same bits as a plain fp32 -> fp16 cast
    assert torch.equal(hi.view(torch.int16), state[:, :, m_lo:].half().view(torch.int16))
    back = sata.join_state(lo, hi, P, dK)
    torch.cuda.synchronize()
    assert torch.equal(back[:, :, :m_lo], state[:, :, :m_lo])
    assert torch.equal(back[:, :, m_lo:], hi.float())


@pytest.mark.parametrize("B,H,dK,dV,P,dt,N0,steps", [
    (2, 3, 32, 32, 4, "bf16", 300, 8),
    (1, 2, 64, 64, 4, "f32", 200, 6),
    (1, 2, 16, 32, 5, "bf16", 150, 6),   # degree-3 and degree-4 rows in fp16
    (3, 1, 32, 64, 2, "f32", 90, 5),     # P = 2: every row fp32, no fp16 array
])
def test_mixed_decode_small(B, H, dK, dV, P, dt, N0, steps):
    q, k, v = make_qkv(B, H, N0 + steps, dK, dV, seed=dK * 31 + P, dtype=dt)
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    _, state = sata.prefill(qc[:, :, :N0].contiguous(), kc[:, :, :N0].contiguous(),
                            vc[:, :, :N0].contiguous(), P)
    lo, hi = sata.split_state(state, P)
    S_or = oracle.final_state(k[:, :, :N0], v[:, :, :N0], P)
    worst = 0.0
    for s in range(steps):
        i = N0 + s
        out = sata.decode_step_mixed(qc[:, :, i].contiguous(), kc[:, :, i].contiguous(),
                                     vc[:, :, i].contiguous(), lo, hi, P)
        ref, S_or = oracle.decode_step(q[:, :, i], k[:, :, i], v[:, :, i], S_or, P)
        worst = max(worst, row_err(out.cpu(), ref))
    S = sata.join_state(lo, hi, P, dK).cpu().double().numpy()
    serr = state_col_error(S, S_or)
    record(f"mixed decode {B}x{H} dK={dK} dV={dV} P={P} {dt}", out_err=worst, state_err=serr,
           excluded_rows=0, rows=B * H * steps, tol=TOL["bf16"], dtype=dt,
           kernels=["decode_bulk", "decode_finalize"])
    assert worst <= TOL["bf16"], worst
    assert serr <= TOL["bf16"], serr


def test_workload5_mixed_decode():
    """Workload 5 on the mixed-precision state: bf16 prefill N=8192 for
    B=32,H=8 (dK=dV=64, P=4), split, then 1024 decode steps.  Two sampled
    heads against the oracle's own trajectory at every step; every head at
    steps 1 and 1024 against the oracle's step from the GPU state before it."""
    w = WORKLOADS[5]
    P = w.P
    q, k, v = workload_inputs(5)
    sample = [(3, 1), (30, 6)]
    _, state = sata.prefill(q.cuda(), k.cuda(), v.cuda(), P)
    lo, hi = sata.split_state(state, P)
    del state
    ks = torch.stack([k[b, h] for b, h in sample])[None]
    vs = torch.stack([v[b, h] for b, h in sample])[None]
    S_or = oracle.final_state(ks, vs, P)
    stream = DecodeStream(5)
    worst = 0.0
    for t in range(1, w.decode_steps + 1):
        qt, kt, vt = stream.next()
        if t in (1, w.decode_steps):
            before = sata.join_state(lo, hi, P, w.dK).cpu()
        out = sata.decode_step_mixed(qt.cuda(), kt.cuda(), vt.cuda(), lo, hi, P)
        o = out.cpu().double().numpy()
        qs_ = np.stack([qt[b, h, 0].double().numpy() for b, h in sample])[None]
        ks_ = np.stack([kt[b, h, 0].double().numpy() for b, h in sample])[None]
        vs_ = np.stack([vt[b, h, 0].double().numpy() for b, h in sample])[None]
        ref, S_or = oracle.decode_step(qs_, ks_, vs_, S_or, P)
        worst = max(worst, row_err(np.stack([o[b, h] for b, h in sample])[None], ref))
        if t in (1, w.decode_steps):
            for b in range(w.B):
                ref_b, _ = oracle.decode_step(qt[b:b + 1, :, 0], kt[b:b + 1, :, 0],
                                              vt[b:b + 1, :, 0], before[b:b + 1], P)
                assert row_err(o[b:b + 1], ref_b) <= TOL["bf16"], (t, b)
            del before
    S = sata.join_state(lo, hi, P, w.dK)
    st_gpu = torch.stack([S[b, h] for b, h in sample])[None].cpu().double().numpy()
    serr = state_col_error(st_gpu, S_or)
    record("workload 5 mixed-precision state (decode B=32,H=8, 1024 steps; heads (3,1),(30,6))",
           out_err=worst, state_err=serr, excluded_rows=0, rows=2 * w.decode_steps,
           tol=TOL["bf16"], dtype="bfloat16", kernels=["decode_bulk", "decode_finalize"])
    assert worst <= TOL["bf16"], worst
    assert serr <= TOL["bf16"], serr
