"""sata_decode_step_noalloc against sata_decode_step (GPU).

The allocation-free decode entry point exists for callers that cannot
allocate device memory: hosts whose caching allocator has reserved the whole
GPU, serving loops that must not call cudaMalloc/cudaFree because those can
synchronise the device, and plug-in hosts whose policy forbids allocations
made by a library.  Its scratch and basis tables are static device arrays, so
it must return what the regular entry point returns, call after call.

This file is named to be collected last: a run that stops at the first failure
has then already run every other test.  It passes alone in a fresh process and
after the other tests, because every call clears the static scratch it uses.
"""
import numpy as np
import pytest
import torch

import linear_cost_attention_b200 as sata
from sata_inputs import make_qkv
from tests.parity import TOL, state_col_error

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from linear_cost_attention_b200 import build

    build.build()
    torch.cuda.set_device(0)


def _row_err(a, b):
    a = a.double().cpu().numpy()
    b = b.double().cpu().numpy()
    return float(np.max(np.max(np.abs(a - b), axis=-1) / np.max(np.abs(b), axis=-1)))


@pytest.mark.parametrize("dt,B,H,dK,dV,P", [
    ("f32", 2, 4, 64, 64, 4),
    ("bf16", 3, 2, 32, 16, 3),
])
def test_noalloc_matches_regular_entry_point_two_calls(dt, B, H, dK, dV, P):
    N0 = 40
    q, k, v = make_qkv(B, H, N0 + 2, dK, dV, seed=77 + dK, dtype=dt)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    _, state = sata.prefill(qd[:, :, :N0].contiguous(), kd[:, :, :N0].contiguous(),
                            vd[:, :, :N0].contiguous(), P)
    s_ref, s_na = state.clone(), state.clone()
    out_ref = torch.empty(B, H, dV, device="cuda")
    out_na = torch.empty(B, H, dV, device="cuda")
    steps = [tuple(t[:, :, N0 + s].contiguous() for t in (qd, kd, vd)) for s in range(2)]
    torch.cuda.synchronize()
    free_after_first = None
    for s, (qt, kt, vt) in enumerate(steps):
        sata.sata_decode_step(qt, kt, vt, s_ref, out_ref, B, H, dK, dV, P, q.dtype)
        sata.sata_decode_step_noalloc(qt, kt, vt, s_na, out_na, B, H, dK, dV, P, q.dtype)
        torch.cuda.synchronize()
        assert _row_err(out_na, out_ref) <= TOL[dt], s
        assert state_col_error(s_na.double().cpu().numpy(),
                               s_ref.double().cpu().numpy()) <= TOL[dt], s
        if s == 0:
            free_after_first = torch.cuda.mem_get_info()[0]
    # the second call allocated nothing (allocation granularity is 2 MiB)
    assert torch.cuda.mem_get_info()[0] > free_after_first - (2 << 20)
    assert sata.sata_get_error() == sata.SATA_OK


def test_noalloc_rejects_sizes_beyond_the_static_scratch():
    L = sata.lib()
    A = 1 << 20  # fake aligned addresses: the size check runs before any device work
    # 1009 heads x 65 columns = 65585 > 65536 partial sums
    st = L.sata_decode_step_noalloc(A, 2 * A, 3 * A, 1 << 40, 4 * A, 1009, 1, 64, 64, 4, 1, None)
    assert st == sata.SATA_ERR_INVALID_ARG
    # 1008 heads fit; with null pointers it still fails, but on the pointer check
    st = L.sata_decode_step_noalloc(None, 2 * A, 3 * A, 1 << 40, 4 * A, 1008, 1, 64, 64, 4, 1,
                                    None)
    assert st == sata.SATA_ERR_INVALID_ARG
