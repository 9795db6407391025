"""Parity of the CUDA path (through the C ABI) with the fp64 oracle on the
seeded workloads, plus edge cases.  Needs a B200."""
import json
import os

import numpy as np
import pytest
import torch

import oracle
import linear_cost_attention_b200 as sata
from sata_inputs import WORKLOADS, DecodeStream, make_qkv, workload_inputs
from tests.parity import TOL, out_row_error, state_col_error

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from linear_cost_attention_b200 import build

    build.build()
    torch.cuda.set_device(0)
    sata.sata_profile_enable(True)  # to report which kernels each call launched
    yield
    sata.sata_profile_enable(False)
    assert sata.sata_get_error() == sata.SATA_OK


def gpu_prefill(q, k, v, P):
    """Prefill through the C ABI into NaN-filled outputs (canaries: every
    element the call must write is checked to have been written)."""
    B, H, N, dK = q.shape
    dV = v.shape[-1]
    m = sata.sata_basis_size(dK, P)
    out = torch.full((B, H, N, dV), float("nan"), device="cuda")
    state = torch.full((B, H, m, dV + 1), float("nan"), device="cuda")
    sata.prefill(q.cuda(), k.cuda(), v.cuda(), P, out=out, state=state)
    torch.cuda.synchronize()
    out, state = out.cpu().double().numpy(), state.cpu().double().numpy()
    assert not np.isnan(state).any(), "state element left unwritten"
    assert not np.isnan(out).any(), "output element left unwritten"
    return out, state


def record(name, **kw):
    """Append the achieved error margins to the file named by SATA_PARITY_LOG."""
    path = os.environ.get("SATA_PARITY_LOG")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps({"case": name, **kw}) + "\n")


def check_prefill(q, k, v, P, tol, heads=None, with_state=True, name=None):
    out, state = gpu_prefill(q, k, v, P)
    if heads is not None:  # oracle on a sample of (b, h) heads
        sel = [(b, h) for b, h in heads]
        qs = torch.stack([q[b, h] for b, h in sel])[None]
        ks = torch.stack([k[b, h] for b, h in sel])[None]
        vs = torch.stack([v[b, h] for b, h in sel])[None]
        out = np.stack([out[b, h] for b, h in sel])[None]
        state = np.stack([state[b, h] for b, h in sel])[None]
        q, k, v = qs, ks, vs
    num, den, ref = oracle.quadratic_form(q, k, v, P)
    cond = oracle.conditioning(q, k, P)
    err, excluded = out_row_error(out, ref, den, cond)
    assert excluded <= max(4, out.shape[-2] * out.shape[0] * out.shape[1] // 200), excluded
    assert err <= tol, (err, tol)
    serr = None
    if with_state:
        S_ref = oracle.final_state(k, v, P)
        serr = state_col_error(state, S_ref)
        assert serr <= tol, (serr, tol)
        # the degree-0 normaliser entry counts tokens exactly
        assert np.all(state[..., 0, -1] == q.shape[2])
    record(name or "prefill %s P=%d" % ("x".join(map(str, q.shape)) + "/" + str(v.shape[-1]), P),
           out_err=err, state_err=serr, excluded_rows=excluded,
           rows=int(np.prod(out.shape[:-1])), tol=tol, dtype=str(q.dtype).split(".")[-1],
           kernels=launched_kernels())
    return err, serr, excluded


def launched_kernels():
    """Names of the kernels the most recent profiled call launched."""
    return sorted({n for n, _ in sata.sata_profile_read()})


def test_workload1_tiny_fp32_full():
    q, k, v = workload_inputs(1)
    out, state = gpu_prefill(q, k, v, 4)
    assert out.shape == (1, 1, 64, 8) and state.shape == (1, 1, 165, 9)
    num, den, ref, S_ref = oracle.feature_form(q, k, v, 4)
    err, excluded = out_row_error(out, ref, den, oracle.conditioning(q, k, 4))
    serr = state_col_error(state, S_ref)
    record("workload 1 (fp32 [1,1,64,8], P=4)", out_err=err, state_err=serr,
           excluded_rows=excluded, rows=64, tol=TOL["f32"], dtype="float32",
           kernels=launched_kernels())
    assert err <= TOL["f32"]
    assert serr <= TOL["f32"]


@pytest.mark.parametrize("P", [4, 3, 2])
def test_workload2_fp32(P):
    q, k, v = workload_inputs(2)
    check_prefill(q, k, v, P, TOL["f32"], name=f"workload 2 (fp32 [2,4,1024,16], P={P})")


def test_workload3_bf16():
    q, k, v = workload_inputs(3)
    check_prefill(q, k, v, 4, TOL["bf16"], name="workload 3 (bf16 [4,8,4096,32], P=4)")
    # bf16 with dK = dV = 32 runs on the tensor cores
    assert {"tc_chunk_states", "tc_readout"} <= set(launched_kernels())


def test_workload4_bf16_sampled_heads():
    q, k, v = workload_inputs(4)
    check_prefill(q, k, v, 4, TOL["bf16"], heads=[(0, 0), (0, 5)],
                  name="workload 4 (bf16 [1,8,16384,64], P=4; heads 0 and 5)")


@pytest.mark.parametrize("B,H,N,dK,dV,P,dt", [
    (1, 1, 1, 8, 8, 4, "f32"),          # a single token
    (1, 2, 77, 16, 8, 4, "f32"),        # ragged tail, dK != dV
    (2, 3, 200, 8, 64, 3, "f32"),
    (1, 1, 1000, 64, 16, 4, "f32"),     # several chunks + ragged tail
    (3, 1, 129, 32, 32, 1, "f32"),      # P = 1: running mean
    (1, 2, 300, 64, 64, 2, "bf16"),
    (2, 2, 1100, 32, 32, 4, "bf16"),
    (2, 2, 150, 8, 16, 5, "f32"),       # P = 5: degree-4 features (495 rows)
    (1, 2, 700, 16, 16, 5, "bf16"),     # P = 5, several chunks (4845 rows)
    (1, 1, 40, 64, 64, 5, "bf16"),      # P = 5 at dK = 64: 814385 rows, CUDA cores
])
def test_edge_shapes(B, H, N, dK, dV, P, dt):
    q, k, v = make_qkv(B, H, N, dK, dV, seed=B * 1000 + N, dtype=dt)
    check_prefill(q, k, v, P, TOL[dt])


@pytest.mark.parametrize("B,H,N", [
    (1, 1, 1),        # one token
    (1, 2, 100),      # ragged, one partial key block
    (1, 1, 128),      # exactly one block, no snapshot
    (2, 1, 1024),     # one chunk, several items per head
    (1, 1, 4096),     # exactly one full chunk, no snapshot
    (1, 2, 4224),     # one snapshot + a block of the next chunk
    (1, 1, 9000),     # two snapshots, ragged tail
])
def test_tensor_core_prefill_shapes(B, H, N):
    # bf16, dK = dV = 64, P = 4: the tcgen05 path
    q, k, v = make_qkv(B, H, N, 64, 64, seed=7 * N + H, dtype="bf16")
    check_prefill(q, k, v, 4, TOL["bf16"])
    assert {"tc_chunk_states", "tc_readout"} <= set(launched_kernels())


@pytest.mark.parametrize("B,H,N", [
    (1, 1, 1),        # one token
    (2, 3, 100),      # ragged, one partial key block
    (1, 2, 1024),     # exactly one full chunk (1024 tokens at dK = 32)
    (1, 1, 1280),     # one snapshot + a block of the next chunk
    (1, 2, 4096),     # four chunks, three snapshots
    (2, 1, 9000),     # eight snapshots, ragged tail
])
def test_tensor_core_prefill_shapes_dk32(B, H, N):
    # bf16, dK = dV = 32, P = 4: the tcgen05 path with 4 index octets and N = 48
    q, k, v = make_qkv(B, H, N, 32, 32, seed=11 * N + H, dtype="bf16")
    check_prefill(q, k, v, 4, TOL["bf16"])
    assert {"tc_chunk_states", "tc_readout"} <= set(launched_kernels())


def test_invalid_call_raises():
    q = torch.zeros(1, 1, 4, 8, device="cuda")
    with pytest.raises(sata.SataError):
        sata.prefill(q, q, q, P=6)
    with pytest.raises(sata.SataError):
        sata.sata_prefill(q, q, q, q, q, 1, 1, 4, 8, 8, 4, torch.float32)  # aliasing


@pytest.mark.parametrize("dt,P", [("f32", 4), ("bf16", 4), ("f32", 5)])
def test_prefill_then_decode_equals_longer_prefill(dt, P):
    B, H, N0, t, dK, dV = 2, 2, 96, 6, 16, 16
    q, k, v = make_qkv(B, H, N0 + t, dK, dV, seed=31, dtype=dt)
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    out_full, state_full = sata.prefill(qc, kc, vc, P)
    _, state = sata.prefill(qc[:, :, :N0].contiguous(), kc[:, :, :N0].contiguous(),
                            vc[:, :, :N0].contiguous(), P)
    outs = []
    for s in range(t):
        i = N0 + s
        outs.append(sata.decode_step(qc[:, :, i].contiguous(), kc[:, :, i].contiguous(),
                                     vc[:, :, i].contiguous(), state, P).cpu())
    torch.cuda.synchronize()
    got = torch.stack(outs, dim=2).double().numpy()
    num, den, ref = oracle.quadratic_form(q, k, v, P)
    cond = oracle.conditioning(q, k, P)
    err, _ = out_row_error(got, ref[:, :, N0:], den[:, :, N0:], cond[:, :, N0:])
    assert err <= TOL[dt]
    tol = TOL[dt]
    assert state_col_error(state.cpu().double().numpy(), oracle.final_state(k, v, P)) <= tol
    # decode continues the GPU prefill consistently with the GPU's longer prefill
    assert state_col_error(state.cpu().double().numpy(),
                           state_full.cpu().double().numpy()) <= 10 * TOL["f32"]


def check_continue(B, H, N0, N1, dK, dV, P, dt, seed):
    """GPU prefill of N0 tokens, then a continued prefill of N1 more: the later
    outputs against the definition over all N0 + N1 tokens, the state against
    the whole sequence's state."""
    q, k, v = make_qkv(B, H, N0 + N1, dK, dV, seed=seed, dtype=dt)
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    _, state = sata.prefill(qc[:, :, :N0].contiguous(), kc[:, :, :N0].contiguous(),
                            vc[:, :, :N0].contiguous(), P)
    out = sata.prefill_continue(qc[:, :, N0:].contiguous(), kc[:, :, N0:].contiguous(),
                                vc[:, :, N0:].contiguous(), state, P)
    torch.cuda.synchronize()
    num, den, ref = oracle.quadratic_form(q, k, v, P)
    cond = oracle.conditioning(q, k, P)
    err, excluded = out_row_error(out.cpu().double().numpy(), ref[:, :, N0:], den[:, :, N0:],
                                  cond[:, :, N0:])
    assert excluded <= max(4, B * H * N1 // 200), excluded
    assert err <= TOL[dt], (err, TOL[dt])
    S = state.cpu().double().numpy()
    assert state_col_error(S, oracle.final_state(k, v, P)) <= TOL[dt]
    assert np.all(S[..., 0, -1] == N0 + N1)


@pytest.mark.parametrize("B,H,N0,N1,dK,dV,P,dt", [
    (2, 2, 300, 500, 16, 8, 4, "f32"),     # CUDA-core path, several chunks after the prefix
    (1, 3, 1, 1, 8, 8, 3, "f32"),          # one token each
    (1, 1, 700, 90, 32, 32, 4, "bf16"),    # CUDA-core path, bf16 inputs
])
def test_prefill_continue(B, H, N0, N1, dK, dV, P, dt):
    check_continue(B, H, N0, N1, dK, dV, P, dt, seed=N0 + 7 * N1)


@pytest.mark.parametrize("N0,N1,d", [
    (4224, 4300, 64),   # prefix with one snapshot; continuation crosses a chunk boundary
    (100, 50, 64),      # short prefix, single-chunk continuation
    (300, 4200, 32),    # dK = dV = 32
])
def test_prefill_continue_tensor_core(N0, N1, d):
    check_continue(1, 2, N0, N1, d, d, 4, "bf16", seed=N0 + N1)


@pytest.mark.parametrize("dt,dK", [("bf16", 64), ("f32", 16)])
def test_prefill_continue_from_zero_is_prefill(dt, dK):
    q, k, v = make_qkv(1, 2, 1500, dK, dK, seed=5, dtype=dt)
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    out0, state0 = sata.prefill(qc, kc, vc, 4)
    state = torch.zeros_like(state0)
    out1 = sata.prefill_continue(qc, kc, vc, state, 4)
    torch.cuda.synchronize()
    torch.testing.assert_close(out1, out0, rtol=1e-5, atol=1e-6)
    torch.testing.assert_close(state, state0, rtol=1e-5, atol=1e-6)


def test_serving_loop_prefill_decode_continue():
    # prompt -> two decode steps -> more prompt -> one decode step, against one
    # pass of the definition over the whole sequence
    N0, N1, P = 200, 150, 4
    q, k, v = make_qkv(2, 2, N0 + 3 + N1, 16, 16, seed=77)
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    outs = []
    o, state = sata.prefill(qc[:, :, :N0].contiguous(), kc[:, :, :N0].contiguous(),
                            vc[:, :, :N0].contiguous(), P)
    outs.append(o)
    for i in (N0, N0 + 1):
        outs.append(sata.decode_step(qc[:, :, i].contiguous(), kc[:, :, i].contiguous(),
                                     vc[:, :, i].contiguous(), state, P)[:, :, None])
    a, b = N0 + 2, N0 + 2 + N1
    outs.append(sata.prefill_continue(qc[:, :, a:b].contiguous(), kc[:, :, a:b].contiguous(),
                                      vc[:, :, a:b].contiguous(), state, P))
    outs.append(sata.decode_step(qc[:, :, b].contiguous(), kc[:, :, b].contiguous(),
                                 vc[:, :, b].contiguous(), state, P)[:, :, None])
    torch.cuda.synchronize()
    got = torch.cat([x.cpu() for x in outs], dim=2).double().numpy()
    num, den, ref = oracle.quadratic_form(q, k, v, P)
    err, _ = out_row_error(got, ref, den, oracle.conditioning(q, k, P))
    assert err <= TOL["f32"], err
    assert state_col_error(state.cpu().double().numpy(), oracle.final_state(k, v, P)) <= TOL["f32"]


def test_workload5_decode():
    """Workload 5: bf16 prefill N=8192 for B=32,H=8 (dK=dV=64, P=4), then 1024
    decode steps.  Oracle: two sampled heads over every step from the oracle's
    own prefill state; all heads at steps 1, 512, 1024 from the GPU's state just
    before the step."""
    w = WORKLOADS[5]
    P = w.P
    q, k, v = workload_inputs(5)
    sample = [(3, 1), (30, 6)]
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    _, state = sata.prefill(qc, kc, vc, P)
    del qc, kc, vc
    ks = torch.stack([k[b, h] for b, h in sample])[None]
    vs = torch.stack([v[b, h] for b, h in sample])[None]
    S_or = oracle.final_state(ks, vs, P)
    st_gpu = torch.stack([state[b, h] for b, h in sample])[None].cpu().double().numpy()
    assert state_col_error(st_gpu, S_or) <= TOL["bf16"]

    stream = DecodeStream(5)
    check_all = {1, 512, 1024}
    worst = 0.0
    for t in range(1, w.decode_steps + 1):
        qt, kt, vt = stream.next()
        if t in check_all:
            before = state.cpu()
        out = sata.decode_step(qt.cuda(), kt.cuda(), vt.cuda(), state, P)
        o = out.cpu().double().numpy()
        # sampled heads against the oracle's own trajectory
        qs_ = np.stack([qt[b, h, 0].double().numpy() for b, h in sample])[None]
        ks_ = np.stack([kt[b, h, 0].double().numpy() for b, h in sample])[None]
        vs_ = np.stack([vt[b, h, 0].double().numpy() for b, h in sample])[None]
        ref, S_or = oracle.decode_step(qs_, ks_, vs_, S_or, P)
        got = np.stack([o[b, h] for b, h in sample])[None]
        e = np.max(np.abs(got - ref), axis=-1) / np.max(np.abs(ref), axis=-1)
        worst = max(worst, float(e.max()))
        if t in check_all:  # every head, from the GPU state before this step
            for b in range(w.B):
                ref_b, _ = oracle.decode_step(qt[b:b + 1, :, 0], kt[b:b + 1, :, 0],
                                              vt[b:b + 1, :, 0], before[b:b + 1], P)
                eb = np.max(np.abs(o[b:b + 1] - ref_b), axis=-1) / np.max(np.abs(ref_b), axis=-1)
                assert eb.max() <= TOL["bf16"], (t, b, eb.max())
            del before
    st_gpu = torch.stack([state[b, h] for b, h in sample])[None].cpu().double().numpy()
    serr = state_col_error(st_gpu, S_or)
    record("workload 5 (decode B=32,H=8, 1024 steps; heads (3,1),(30,6) every step)",
           out_err=worst, state_err=serr, excluded_rows=0, rows=2 * w.decode_steps,
           tol=TOL["bf16"], dtype="bfloat16", kernels=launched_kernels())
    assert worst <= TOL["bf16"], worst
    assert serr <= TOL["bf16"]


def test_p5_decode_dk64_against_oracle():
    """P = 5 at dK = dV = 64 (degree-4 features, 814385 rows, 212 MB of state
    per head): prefill on the CUDA cores, then decode steps, each against the
    oracle's decode step continued from the oracle's own state."""
    B, H, N0, P, steps = 1, 2, 40, 5, 3
    q, k, v = make_qkv(B, H, N0 + steps, 64, 64, seed=555, dtype="bf16")
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    _, state = sata.prefill(qc[:, :, :N0].contiguous(), kc[:, :, :N0].contiguous(),
                            vc[:, :, :N0].contiguous(), P)
    S_or = oracle.final_state(k[:, :, :N0], v[:, :, :N0], P)
    worst = 0.0
    for s in range(steps):
        i = N0 + s
        out = sata.decode_step(qc[:, :, i].contiguous(), kc[:, :, i].contiguous(),
                               vc[:, :, i].contiguous(), state, P)
        ref, S_or = oracle.decode_step(q[:, :, i], k[:, :, i], v[:, :, i], S_or, P)
        o = out.cpu().double().numpy()
        e = np.max(np.abs(o - ref), axis=-1) / np.max(np.abs(ref), axis=-1)
        worst = max(worst, float(e.max()))
    serr = state_col_error(state.cpu().double().numpy(), S_or)
    record("decode P=5 dK=dV=64 (B=1,H=2, 40-token prefill + 3 steps)", out_err=worst,
           state_err=serr, excluded_rows=0, rows=B * H * steps, tol=TOL["bf16"],
           dtype="bfloat16", kernels=launched_kernels())
    assert worst <= TOL["bf16"], worst
    assert serr <= TOL["bf16"], serr
