"""Host-side checks of the C-ABI library (no GPU): it loads, exports every
symbol include/sata.h declares, its index tables match the oracle bit for bit,
and invalid calls are rejected before anything touches a device."""
import ctypes
import math
import os
import re

import numpy as np
import pytest

import oracle
import linear_cost_attention_b200 as sata

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def built_lib():
    from linear_cost_attention_b200 import build

    build.build()
    return sata.lib()


def _declared_functions():
    names = []
    for h in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if h.endswith(".h"):
            txt = open(os.path.join(ROOT, "include", h)).read()
            txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
            names += re.findall(r"\b(sata_[a-z0-9_]+)\s*\(", txt)
    return sorted(set(names))


def test_every_declared_symbol_is_exported():
    names = _declared_functions()
    assert {"sata_prefill", "sata_decode_step", "sata_basis_size", "sata_index_table"} <= set(names)
    so = ctypes.CDLL(sata.LIB_PATH)
    for n in names:
        assert hasattr(so, n), f"{n} declared in include/ but not exported"


@pytest.mark.parametrize("dK", [1, 3, 8, 16, 32, 64])
@pytest.mark.parametrize("P", [1, 2, 3, 4])
def test_basis_size(dK, P):
    assert sata.sata_basis_size(dK, P) == math.comb(dK + P - 1, P - 1) == oracle.basis_total(dK, P)


def test_basis_size_invalid():
    assert sata.sata_basis_size(0, 4) == -1
    assert sata.sata_basis_size(8, 0) == -1


@pytest.mark.parametrize("dK", [2, 8, 16, 32, 64])
@pytest.mark.parametrize("p", [0, 1, 2, 3])
def test_index_table_bit_exact(dK, p):
    got = sata.sata_index_table(dK, p)
    ref = oracle.basis_rows(dK, p)
    assert got.dtype == np.int32 and got.shape == ref.shape
    assert np.array_equal(got, ref)


def test_index_table_degree4_bit_exact():
    for dK in (3, 8, 16):
        assert np.array_equal(sata.sata_index_table(dK, 4), oracle.basis_rows(dK, 4))


def test_index_table_capacity_and_args():
    L = sata.lib()
    buf = (ctypes.c_int32 * 10)()
    assert L.sata_index_table(8, 2, buf, 10) == -1          # 36 rows x 2 do not fit
    assert L.sata_index_table(8, 2, None, 1000) == -1
    assert L.sata_index_table(0, 2, buf, 10) == -1
    assert L.sata_index_table(8, 0, None, 0) == 1           # one empty row


def test_status_strings():
    for s in range(6):
        assert sata.sata_status_string(s).startswith("SATA_")
    assert "unknown" in sata.sata_status_string(99)


def test_invalid_calls_rejected_on_host():
    L = sata.lib()
    A = 1 << 20  # fake, 16-byte aligned, never dereferenced: validation runs first
    args = dict(B=1, H=1, N=8, dK=8, dV=8, P=4, dt=0)

    def pre(q=A, k=2 * A, v=3 * A, out=4 * A, st=5 * A, **kw):
        a = {**args, **kw}
        return L.sata_prefill(q, k, v, out, st, a["B"], a["H"], a["N"], a["dK"], a["dV"],
                              a["P"], a["dt"], None)

    assert pre(q=None) == sata.SATA_ERR_INVALID_ARG
    assert pre(out=None) == sata.SATA_ERR_INVALID_ARG
    assert pre(k=A + 4) == sata.SATA_ERR_INVALID_ARG            # misaligned
    assert pre(N=0) == sata.SATA_ERR_INVALID_ARG
    assert pre(B=-1) == sata.SATA_ERR_INVALID_ARG
    assert pre(dt=7) == sata.SATA_ERR_INVALID_ARG
    assert pre(dK=12) == sata.SATA_ERR_UNSUPPORTED
    assert pre(dV=128) == sata.SATA_ERR_UNSUPPORTED
    assert pre(P=6) == sata.SATA_ERR_UNSUPPORTED
    assert pre(P=0) == sata.SATA_ERR_UNSUPPORTED
    assert pre(out=A) == sata.SATA_ERR_INVALID_ARG               # out aliases q
    assert pre(st=4 * A + 16) == sata.SATA_ERR_INVALID_ARG        # state overlaps out
    assert pre(N=1 << 30, B=4) == sata.SATA_ERR_INVALID_ARG      # index range

    def cont(q=A, k=2 * A, v=3 * A, out=4 * A, st=5 * A, **kw):
        a = {**args, **kw}
        return L.sata_prefill_continue(q, k, v, out, st, a["B"], a["H"], a["N"], a["dK"],
                                       a["dV"], a["P"], a["dt"], None)

    assert cont(st=None) == sata.SATA_ERR_INVALID_ARG
    assert cont(v=3 * A + 8) == sata.SATA_ERR_INVALID_ARG        # misaligned
    assert cont(P=6) == sata.SATA_ERR_UNSUPPORTED
    assert cont(st=4 * A + 16) == sata.SATA_ERR_INVALID_ARG       # state overlaps out

    def dec(q=A, k=2 * A, v=3 * A, st=5 * A, out=4 * A, **kw):
        a = {**args, **kw}
        return L.sata_decode_step(q, k, v, st, out, a["B"], a["H"], a["dK"], a["dV"], a["P"],
                                  a["dt"], None)

    assert dec(v=None) == sata.SATA_ERR_INVALID_ARG
    assert dec(st=5 * A + 8) == sata.SATA_ERR_INVALID_ARG
    assert dec(H=0) == sata.SATA_ERR_INVALID_ARG
    assert dec(dK=7) == sata.SATA_ERR_UNSUPPORTED
    assert dec(out=2 * A) == sata.SATA_ERR_INVALID_ARG
    # head and output indices are 32-bit in the kernels: B*H*(dV+1) < 2^31
    assert dec(B=1 << 25, P=1, dV=64) == sata.SATA_ERR_INVALID_ARG


def test_plain_c_program_uses_the_abi(tmp_path):
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    sata.lib()  # builds or finds the in-tree library
    libdir = os.path.dirname(sata.LIB_PATH)
    exe = tmp_path / "abi_c_check"
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "cpu", "abi_c_check.c"), "-o", str(exe),
                    "-L", libdir, "-lsata", f"-Wl,-rpath,{libdir}"], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == "ok", (r.returncode, r.stdout, r.stderr)


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    import importlib

    monkeypatch.setattr(sata, "_lib", None)
    monkeypatch.setattr(sata, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="missing"):
        sata.lib()


def test_mixed_state_calls_rejected_on_host():
    L = sata.lib()
    A = 1 << 20
    assert L.sata_state_fp32_rows(64, 4) == 2145 == math.comb(66, 2)
    assert L.sata_state_fp32_rows(64, 2) == 65
    assert L.sata_state_fp32_rows(0, 4) == -1
    # hi array required when P >= 4 has fp16 rows
    assert L.sata_state_split(A, 2 * A, None, 1, 1, 8, 8, 4, None) == sata.SATA_ERR_INVALID_ARG
    assert L.sata_state_split(A, 2 * A + 8, 3 * A, 1, 1, 8, 8, 4, None) == sata.SATA_ERR_INVALID_ARG
    assert L.sata_state_join(A, 3 * A, A, 1, 1, 8, 8, 4, None) == sata.SATA_ERR_INVALID_ARG
    assert L.sata_state_split(A, 2 * A, 3 * A, 1, 1, 12, 8, 4, None) == sata.SATA_ERR_UNSUPPORTED
    dm = L.sata_decode_step_mixed
    assert dm(A, 2 * A, 3 * A, 4 * A, 5 * A, 6 * A, 1, 1, 8, 16, 4, 1, None) == \
        sata.SATA_ERR_UNSUPPORTED                                 # dV = 16: no bulk kernel
    assert dm(A, 2 * A, 3 * A, 4 * A, None, 6 * A, 1, 1, 8, 32, 4, 1, None) == \
        sata.SATA_ERR_INVALID_ARG                                 # missing fp16 array
    assert dm(A, 2 * A, 3 * A, 4 * A, 5 * A, A, 1, 1, 8, 32, 4, 1, None) == \
        sata.SATA_ERR_INVALID_ARG                                 # out aliases q


def test_backward_call_rejected_on_host():
    L = sata.lib()
    A = 1 << 20
    bw = L.sata_attention_backward
    args = (1, 1, 8, 8, 8, 4, 0, None)
    # every call below must fail validation: nothing may reach a launch
    assert bw(None, 2 * A, 3 * A, 4 * A, 5 * A, 6 * A, 7 * A, *args) == sata.SATA_ERR_INVALID_ARG
    assert bw(A, 2 * A, 3 * A, 4 * A, 5 * A + 4, 6 * A, 7 * A, *args) == sata.SATA_ERR_INVALID_ARG
    assert bw(A, 2 * A, 3 * A, 4 * A, A, 6 * A, 7 * A, *args) == sata.SATA_ERR_INVALID_ARG  # dq = q
    assert bw(A, 2 * A, 3 * A, 4 * A, 5 * A, 5 * A, 7 * A, *args) == sata.SATA_ERR_INVALID_ARG
    assert bw(A, 2 * A, 3 * A, 4 * A, 5 * A, 6 * A, 7 * A, 1, 1, 8, 12, 8, 4, 0, None) == \
        sata.SATA_ERR_UNSUPPORTED
