"""Failure detection on the GPU without a fault: the tensor-core prefill's
bounded waits are made to run out (test hook ``sata_test_set_wait_limit``),
the call must return, ``sata_get_error`` must report SATA_ERR_TIMEOUT, and the
device must stay usable: the next normal prefill passes parity.  No wait is
left unbounded and nothing traps: a role whose wait runs out records the
error, the CTA's other roles leave their loops, and every CTA still drains its
own copies and MMAs (with the default bound) before it frees its TMEM."""
import numpy as np
import pytest
import torch

import oracle
import linear_cost_attention_b200 as sata
from sata_inputs import make_qkv
from tests.parity import TOL, out_row_error, state_col_error

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from linear_cost_attention_b200 import build

    build.build()
    torch.cuda.set_device(0)
    yield
    sata.sata_test_set_wait_limit(0)


def test_wait_that_runs_out_reports_timeout_and_device_recovers():
    # bf16, dK = dV = 64, P = 4 (tensor-core path), two chunk-boundary snapshots
    q, k, v = make_qkv(1, 2, 9000, 64, 64, seed=91, dtype="bf16")
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    assert sata.sata_get_error() == sata.SATA_OK
    prev = sata.sata_test_set_wait_limit(1)  # every role wait that is not met at once gives up
    try:
        sata.prefill(qc, kc, vc, 4)  # returns: launches are asynchronous
        status = sata.sata_get_error()  # synchronises: the kernels have finished
    finally:
        sata.sata_test_set_wait_limit(prev)
    assert status == sata.SATA_ERR_TIMEOUT, sata.sata_status_string(status)
    assert sata.sata_get_error() == sata.SATA_OK  # reported once, then cleared

    # the context is intact: a normal call on the same inputs passes parity
    out, state = sata.prefill(qc, kc, vc, 4)
    torch.cuda.synchronize()
    assert sata.sata_get_error() == sata.SATA_OK
    num, den, ref = oracle.quadratic_form(q, k, v, 4)
    err, excluded = out_row_error(out.cpu().double().numpy(), ref, den,
                                  oracle.conditioning(q, k, 4))
    assert excluded <= 2 * 9000 // 200
    assert err <= TOL["bf16"], err
    S = state.cpu().double().numpy()
    assert state_col_error(S, oracle.final_state(k, v, 4)) <= TOL["bf16"]
    assert np.all(S[..., 0, -1] == 9000)
