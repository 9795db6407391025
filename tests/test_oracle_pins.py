"""Pins of the fp64 oracle against what the pages and mathematics fix (CPU only).

Each test names the fact it pins.  None re-types the oracle's own formula: the
checks are closed forms, page values, brute force over the full expansion,
special cases that reduce to textbook computations, and invariances.
"""
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
from oracle import basis as obasis
from oracle import brute
from sata_inputs import make_qkv, workload_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "page_values.txt")


def _golden():
    vals = {}
    with open(GOLDEN) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            name, *kv, value = line.split()
            vals[(name, tuple(kv))] = int(value)
    return vals


def _rng(seed=0):
    return np.random.default_rng(seed)


# ---------------------------------------------------------------- basis tables

@pytest.mark.parametrize("dK", [1, 2, 3, 5, 8, 16, 32, 64])
@pytest.mark.parametrize("p", [0, 1, 2, 3])
def test_basis_count_is_multiset_coefficient(dK, p):
    # [SATA-eng] "对称张量分解的核心洞察": minimal basis size C(d_K+p-1, p).
    assert len(obasis.basis_rows(dK, p)) == math.comb(dK + p - 1, p)


def test_basis_count_degree4_small():
    for dK in (2, 3, 7, 12):
        assert len(obasis.basis_rows(dK, 4)) == math.comb(dK + 3, 4)


def test_page_basis_total_47905():
    g = _golden()
    assert oracle.basis_total(64, 4) == g[("basis_total", ("dK=64", "P=4"))] == 47905
    # hockey-stick identity: sum_{p<P} C(dK+p-1,p) = C(dK+P-1, P-1)
    for dK in (8, 16, 32, 64):
        assert oracle.basis_total(dK, 4) == math.comb(dK + 3, 3)


def test_page_full_expansion_size():
    g = _golden()
    bound = g[("full_expansion_lower_bound", ("dK=64", "p=4"))]
    assert 64 ** 4 > bound
    assert len(obasis.basis_rows(16, 4)) < 16 ** 4 // 10


@pytest.mark.parametrize("dK,p", [(8, 3), (16, 3), (64, 3), (5, 4)])
def test_rows_sorted_and_lexicographic(dK, p):
    rows = obasis.basis_rows(dK, p)
    assert rows.dtype == np.int32
    assert (rows >= 0).all() and (rows < dK).all()
    assert (np.diff(rows, axis=1) >= 0).all()              # i1 <= i2 <= ... <= ip
    tuples = [tuple(r) for r in rows]
    assert all(a < b for a, b in zip(tuples, tuples[1:]))   # strictly increasing lex
    # every sorted tuple appears exactly once (distinct and complete)
    assert len(set(tuples)) == len(tuples) == math.comb(dK + p - 1, p)


@pytest.mark.parametrize("dK", [2, 3, 8, 16])
@pytest.mark.parametrize("p", [1, 2, 3, 4])
def test_multinomial_theorem(dK, p):
    # sum over sorted tuples of p!/alpha! equals the number of ordered tuples dK^p
    rows = obasis.basis_rows(dK, p)
    total = sum(math.factorial(p) // obasis.multiplicity_factorial(r) for r in rows)
    assert total == dK ** p


def test_weight_spot_values():
    w = obasis.basis_weights(64, 3, np.array([[0, 0, 0], [0, 0, 1], [0, 1, 2]], np.int32))
    # alpha! = 6, 2, 1; d_K^(3/2) = 512
    np.testing.assert_allclose(w, [1 / math.sqrt(3072), 1 / math.sqrt(1024), 1 / math.sqrt(512)],
                               rtol=0, atol=1e-15)
    assert obasis.basis_weights(64, 0)[0] == 1.0


@pytest.mark.parametrize("dK", [3, 8, 16, 64])
@pytest.mark.parametrize("p", [0, 1, 2, 3])
def test_feature_kernel_identity_per_degree(dK, p):
    # sum over the degree-p block of phi(q) phi(k) = (q.k / sqrt(dK))^p / p!
    r = _rng(dK * 10 + p)
    q = r.standard_normal(dK)
    k = r.standard_normal(dK)
    basis = [(p, obasis.basis_rows(dK, p), obasis.basis_weights(dK, p))]
    lhs = float(oracle.feature_map(q, p + 1, basis) @ oracle.feature_map(k, p + 1, basis))
    s = float(q @ k) / math.sqrt(dK)
    rhs = s ** p / math.factorial(p)
    assert abs(lhs - rhs) <= 1e-13 * max(1.0, abs(rhs))


def test_taylor_kernel_values():
    # closed forms: T_4(1) = 8/3, T_4(-2) = -1/3, T_1 = 1, T_2(s) = 1 + s
    assert abs(oracle.taylor_kernel(1.0, 4) - 8 / 3) < 1e-15
    assert abs(oracle.taylor_kernel(-2.0, 4) + 1 / 3) < 1e-15
    assert oracle.taylor_kernel(5.0, 1) == 1.0
    assert oracle.taylor_kernel(0.25, 2) == 1.25
    # converges to exp as P grows
    assert abs(oracle.taylor_kernel(0.7, 25) - math.exp(0.7)) < 1e-15


# ------------------------------------------------------ attention computations

def _rowerr(a_num, a_den, b_num, b_den):
    a = np.concatenate([a_num, a_den[..., None]], axis=-1)
    b = np.concatenate([b_num, b_den[..., None]], axis=-1)
    return float(np.max(np.max(np.abs(a - b), axis=-1) / np.max(np.abs(b), axis=-1)))


@pytest.mark.parametrize("dK,P,N", [(2, 1, 5), (2, 2, 9), (2, 4, 12), (3, 3, 10), (4, 4, 8)])
def test_brute_force_full_expansion(dK, P, N):
    r = _rng(dK * 100 + P * 10 + N)
    q = r.standard_normal((1, 1, N, dK))
    k = r.standard_normal((1, 1, N, dK))
    v = r.standard_normal((1, 1, N, 3))
    bn, bd = brute.brute_attention(q[0, 0], k[0, 0], v[0, 0], P)
    an, ad, _ = oracle.quadratic_form(q, k, v, P)
    fn, fd, _, _ = oracle.feature_form(q, k, v, P)
    assert _rowerr(an[0, 0], ad[0, 0], bn, bd) < 1e-12
    assert _rowerr(fn[0, 0], fd[0, 0], bn, bd) < 1e-12


@pytest.mark.parametrize("wid", [1, 2])
def test_quadratic_and_feature_forms_agree(wid):
    q, k, v = workload_inputs(wid)
    an, ad, _ = oracle.quadratic_form(q, k, v, 4)
    fn, fd, _, _ = oracle.feature_form(q, k, v, 4)
    assert _rowerr(fn, fd, an, ad) < 1e-10


def test_hand_worked_example():
    # d_K = 4 (sqrt = 2), d_V = 1, P = 4, three tokens, computed by hand in fractions.
    q = np.array([[0, 0, 0, 0], [1, 0.5, 0, 0], [-2, 0, 0, 0]], float)[None, None]
    k = np.array([[2, 0, 0, 0], [0, 2, 0, 0], [2, 0, 0, 0]], float)[None, None]
    v = np.array([[3], [-1], [5]], float)[None, None]

    def T4(s):
        s = Fraction(s)
        return 1 + s + s * s / 2 + s * s * s / 6

    # token 0: s00 = 0 -> T = 1 -> out = v0
    # token 1: s10 = (1*2)/2 = 1, s11 = (0.5*2)/2 = 1/2
    # token 2: s20 = (-2*2)/2 = -2, s21 = 0, s22 = -2
    t = {(0, 0): T4(0), (1, 0): T4(1), (1, 1): T4(Fraction(1, 2)),
         (2, 0): T4(-2), (2, 1): T4(0), (2, 2): T4(-2)}
    vv = [3, -1, 5]
    num = [sum(t[(i, j)] * vv[j] for j in range(i + 1)) for i in range(3)]
    den = [sum(t[(i, j)] for j in range(i + 1)) for i in range(3)]
    assert t[(1, 0)] == Fraction(8, 3) and t[(1, 1)] == Fraction(79, 48) and t[(2, 0)] == Fraction(-1, 3)
    an, ad, ao = oracle.quadratic_form(q, k, v, 4)
    fn, fd, fo, _ = oracle.feature_form(q, k, v, 4)
    for i in range(3):
        for got_n, got_d in ((an, ad), (fn, fd)):
            assert abs(got_n[0, 0, i, 0] - float(num[i])) < 1e-14
            assert abs(got_d[0, 0, i] - float(den[i])) < 1e-14
    assert abs(ao[0, 0, 1, 0] - 305 / 207) < 1e-14
    assert abs(ao[0, 0, 2, 0] - float(num[2] / den[2])) < 1e-13


def test_P1_is_running_mean():
    q, k, v = make_qkv(1, 2, 40, 8, 5, seed=7)
    _, _, out = oracle.quadratic_form(q, k, v, 1)
    _, _, fo, _ = oracle.feature_form(q, k, v, 1)
    vv = v.double().numpy()
    mean = np.cumsum(vv, axis=2) / np.arange(1, 41)[None, None, :, None]
    np.testing.assert_allclose(out, mean, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(fo, mean, rtol=1e-13, atol=1e-13)


def test_P2_is_textbook_linear_attention():
    # T_2(s) = 1 + s  <=>  linear attention with phi(x) = [1, x / dK^(1/4)]
    B, H, N, dK, dV = 1, 2, 50, 16, 4
    q, k, v = make_qkv(B, H, N, dK, dV, seed=11)
    qq, kk, vv = (t.double().numpy() for t in (q, k, v))
    c = dK ** -0.25
    fq = np.concatenate([np.ones((B, H, N, 1)), qq * c], axis=-1)
    fk = np.concatenate([np.ones((B, H, N, 1)), kk * c], axis=-1)
    kv = np.cumsum(fk[..., :, None] * vv[..., None, :], axis=2)      # [B,H,N,1+dK,dV]
    z = np.cumsum(fk, axis=2)
    ref_num = np.einsum("bhnf,bhnfd->bhnd", fq, kv)
    ref_den = np.einsum("bhnf,bhnf->bhn", fq, z)
    an, ad, _ = oracle.quadratic_form(q, k, v, 2)
    fn, fd, _, _ = oracle.feature_form(q, k, v, 2)
    assert _rowerr(an, ad, ref_num, ref_den) < 1e-12
    assert _rowerr(fn, fd, ref_num, ref_den) < 1e-12


def test_state_structure_closed_forms():
    B, H, N, dK, dV, P = 2, 1, 37, 8, 3, 4
    q, k, v = make_qkv(B, H, N, dK, dV, seed=3)
    _, _, _, S = oracle.feature_form(q, k, v, P)
    kk, vv = k.double().numpy(), v.double().numpy()
    m = math.comb(dK + P - 1, P - 1)
    # [SATA-eng] "恒定计算成本的工程实现": state (d_V+1) x C(d_K+P-1, P-1)
    assert S.shape == (B, H, m, dV + 1)
    # degree-0 row: [sum_j v_j, N]; the normaliser entry is exactly N
    assert (S[:, :, 0, dV] == N).all()
    np.testing.assert_allclose(S[:, :, 0, :dV], vv.sum(axis=2), rtol=1e-13, atol=1e-13)
    # degree-1 rows i: sum_j k_j[i] [v_j, 1] / dK^(1/4)
    v1 = np.concatenate([vv, np.ones((B, H, N, 1))], axis=-1)
    deg1 = np.einsum("bhni,bhnc->bhic", kk, v1) * dK ** -0.25
    np.testing.assert_allclose(S[:, :, 1:1 + dK], deg1, rtol=1e-12, atol=1e-12)
    # matrix-product form of the token sum gives the same state
    np.testing.assert_allclose(oracle.final_state(k, v, P), S, rtol=1e-11, atol=1e-11)


def test_state_size_independent_of_N():
    shapes = set()
    for N in (1, 16, 64, 200):
        q, k, v = make_qkv(1, 1, N, 8, 8, seed=N)
        shapes.add(oracle.feature_form(q, k, v, 4)[3].shape)
    assert shapes == {(1, 1, 165, 9)}


def test_joint_permutation_invariance():
    q, k, v = make_qkv(1, 2, 64, 16, 16, seed=5)
    perm = np.random.default_rng(1).permutation(16)
    _, _, o1 = oracle.quadratic_form(q, k, v, 4)
    _, _, o2 = oracle.quadratic_form(q[..., perm], k[..., perm], v, 4)
    np.testing.assert_allclose(o1, o2, rtol=1e-11, atol=1e-12)
    _, _, f2, _ = oracle.feature_form(q[..., perm], k[..., perm], v, 4)
    np.testing.assert_allclose(o1, f2, rtol=1e-9, atol=1e-10)


def test_decode_continues_prefill():
    N0, t = 24, 5
    q, k, v = make_qkv(2, 2, N0 + t, 8, 8, seed=9)
    _, _, _, S = oracle.feature_form(q[:, :, :N0], k[:, :, :N0], v[:, :, :N0], 4)
    _, _, full_out = oracle.quadratic_form(q, k, v, 4)
    S_ref = oracle.feature_form(q, k, v, 4)[3]
    for s in range(t):
        i = N0 + s
        out, S = oracle.decode_step(q[:, :, i], k[:, :, i], v[:, :, i], S, 4)
        np.testing.assert_allclose(out, full_out[:, :, i], rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(S, S_ref, rtol=1e-12, atol=1e-12)


def test_feature_form_continues_from_a_state():
    # a continued prefill: the per-token procedure started from the state of
    # the first N0 tokens gives, for the later tokens, the definition's rows
    # over the whole sequence, and the whole sequence's state
    N0, N1 = 20, 17
    q, k, v = make_qkv(2, 3, N0 + N1, 8, 4, seed=21)
    S0 = oracle.final_state(k[:, :, :N0], v[:, :, :N0], 4)
    num, den, out, S = oracle.feature_form(q[:, :, N0:], k[:, :, N0:], v[:, :, N0:], 4, state0=S0)
    num_f, den_f, out_f = oracle.quadratic_form(q, k, v, 4)
    np.testing.assert_allclose(num, num_f[:, :, N0:], rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(den, den_f[:, :, N0:], rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(S, oracle.final_state(k, v, 4), rtol=1e-12, atol=1e-12)
    # from a zero state it is the plain prefill
    z = oracle.feature_form(q, k, v, 4, state0=np.zeros_like(S))
    np.testing.assert_allclose(z[2], out_f, rtol=1e-10, atol=1e-12)


def test_softmax_reference_matches_library_attention():
    # the exact-softmax reference used by the error-vs-P pin is PyTorch's own
    # causal scaled dot-product attention (same 1/sqrt(dK) scale), in fp64
    import torch
    q, k, v = make_qkv(2, 3, 70, 16, 8, seed=13)
    ref = torch.nn.functional.scaled_dot_product_attention(
        q.double(), k.double(), v.double(), is_causal=True).numpy()
    np.testing.assert_allclose(oracle.softmax_attention(q, k, v, row_block=32), ref,
                               rtol=1e-12, atol=1e-13)


def test_conditioning_is_the_sum_of_absolute_kernel_values():
    # brute force over (i, j <= i) with the scalar Taylor sum
    q, k, _ = make_qkv(1, 2, 23, 4, 4, seed=17)
    qd, kd = q.double().numpy(), k.double().numpy()
    got = oracle.conditioning(q, k, 4, row_block=5)
    for h in range(2):
        for i in range(23):
            want = 0.0
            for j in range(i + 1):
                s = float(qd[0, h, i] @ kd[0, h, j]) / 2.0
                want += abs(1 + s + s * s / 2 + s ** 3 / 6)
            assert abs(got[0, h, i] - want) <= 1e-12 * want


def test_error_against_softmax_shrinks_with_P():
    # [SATA-eng] "精度与效率的权衡参数": a higher truncation order is more accurate.
    q, k, v = workload_inputs(2)
    q, k, v = q[:1, :2], k[:1, :2], v[:1, :2]
    ref = oracle.softmax_attention(q, k, v)
    errs = []
    for P in (2, 3, 4, 5):
        _, _, out = oracle.quadratic_form(q, k, v, P)
        d = (out - ref)[:, :, 16:]
        errs.append(np.linalg.norm(d) / np.linalg.norm(ref[:, :, 16:]))
    assert errs[0] > errs[1] > errs[2] > errs[3], errs
    # kernel level on the same scores
    qq, kk = q.double().numpy()[0, 0], k.double().numpy()[0, 0]
    s = (qq @ kk.T) / 4.0
    s = s[np.tril_indices(s.shape[0])]
    kerr = [np.mean(np.abs(oracle.taylor_kernel(s, P) - np.exp(s)) / np.exp(s)) for P in (2, 3, 4, 5)]
    assert kerr[0] > kerr[1] > kerr[2] > kerr[3]


@pytest.mark.parametrize("dK,P", [(8, 2), (8, 4), (16, 3), (32, 4), (64, 4), (64, 5)])
def test_page_flop_formula(dK, P):
    # [SATA-eng] "恒定计算成本的工程实现": (4 d_V + 2(P d_K + 1)/(d_K + 1) + 2) C(d_K+P-1, P-1)
    dV = dK
    page = Fraction(4 * dV) + Fraction(2 * (P * dK + 1), dK + 1) + 2
    page *= math.comb(dK + P - 1, P - 1)
    assert page.denominator == 1
    assert oracle.flops_per_token_counted(dK, dV, P) == page.numerator


# ------------------------------------------------- the pins catch planted bugs

def test_pins_catch_planted_mistakes():
    """Plant plausible mistakes in copies of the oracle's pieces (on the CPU) and
    check that a pin above would fail for each."""
    r = _rng(42)
    dK = 8
    q = r.standard_normal(dK)
    k = r.standard_normal(dK)
    s = float(q @ k) / math.sqrt(dK)

    def kernel_via(basis):
        return float(oracle.feature_map(q, 4, basis) @ oracle.feature_map(k, 4, basis))

    good = obasis.basis_all(dK, 4)
    assert abs(kernel_via(good) - oracle.taylor_kernel(s, 4)) < 1e-12
    # (1) weights without the multinomial factor
    bad_w = [(p, rows, np.full(len(rows), dK ** (-p / 4) / math.sqrt(math.factorial(p))))
             for p, rows, _ in good]
    assert abs(kernel_via(bad_w) - oracle.taylor_kernel(s, 4)) > 1e-3
    # (2) dropped degree-0 term
    assert abs(kernel_via(good[1:]) - oracle.taylor_kernel(s, 4)) > 0.5
    # (3) a wrong index in the table
    rows3 = good[3][1].copy()
    rows3[5, 2] = (rows3[5, 2] + 1) % dK
    bad_idx = good[:3] + [(3, rows3, good[3][2])]
    # (the identity pin holds the sum to 1e-13 relative)
    assert abs(kernel_via(bad_idx) - oracle.taylor_kernel(s, 4)) > 1e-10
    # (4) a sign error in the weights cancels in phi(q).phi(k) but not in the
    #     state: the degree-1 closed form of test_state_structure_closed_forms fails
    bad_sign = good[:1] + [(1, good[1][1], -good[1][2])] + good[2:]
    assert abs(kernel_via(bad_sign) - oracle.taylor_kernel(s, 4)) < 1e-12
    kk = r.standard_normal((5, dK))
    vv1 = np.concatenate([r.standard_normal((5, 2)), np.ones((5, 1))], axis=1)
    S_bad = oracle.feature_map(kk, 4, bad_sign).T @ vv1
    deg1 = kk.T @ vv1 * dK ** -0.25
    assert np.max(np.abs(S_bad[1:1 + dK] - deg1)) > 1e-3
    #     and a sign error in the Taylor sum is caught by the brute force
    t_bad = sum((-s) ** p / math.factorial(p) for p in range(4))
    assert abs(t_bad - kernel_via(good)) > 1e-3
    # (5) swapped q and k in the causal sum changes the outputs (and is caught by brute force)
    qq = r.standard_normal((1, 1, 6, 2))
    kk = r.standard_normal((1, 1, 6, 2))
    vv = r.standard_normal((1, 1, 6, 2))
    bn, bd = brute.brute_attention(qq[0, 0], kk[0, 0], vv[0, 0], 3)
    sn, sd, _ = oracle.quadratic_form(kk, qq, vv, 3)
    assert _rowerr(sn[0, 0], sd[0, 0], bn, bd) > 1e-6


# ---------------------------------------------------------------- backward pass

def _loss(q, k, v, dout, P):
    return float((oracle.quadratic_form(q, k, v, P)[2] * dout).sum())


@pytest.mark.parametrize("P", [2, 3, 4, 5])
def test_gradient_matches_finite_differences(P):
    # central differences of the definition itself (a computation independent
    # of the chain rule in attention_grad), element by element
    r = _rng(40 + P)
    B, H, N, dK, dV = 1, 2, 6, 3, 2
    q, k, v = (r.standard_normal((B, H, N, d)) for d in (dK, dK, dV))
    dout = r.standard_normal((B, H, N, dV))
    dq, dk, dv = oracle.attention_grad(q, k, v, dout, P)
    eps = 1e-6
    for x, g in ((q, dq), (k, dk), (v, dv)):
        fd = np.zeros_like(x)
        for idx in np.ndindex(*x.shape):
            old = x[idx]
            x[idx] = old + eps
            lp = _loss(q, k, v, dout, P)
            x[idx] = old - eps
            lm = _loss(q, k, v, dout, P)
            x[idx] = old
            fd[idx] = (lp - lm) / (2 * eps)
        assert np.max(np.abs(fd - g)) <= 1e-6 * max(1.0, np.max(np.abs(g))), np.max(np.abs(fd - g))


def test_gradient_P1_closed_form():
    # P = 1: out_i = mean(v_0..v_i) does not depend on q, k, and
    # dv_j = sum_{i >= j} dout_i / (i + 1)
    r = _rng(77)
    q, k, v = (r.standard_normal((1, 1, 7, 4)) for _ in range(3))
    dout = r.standard_normal((1, 1, 7, 4))
    dq, dk, dv = oracle.attention_grad(q, k, v, dout, 1)
    assert np.all(dq == 0) and np.all(dk == 0)
    want = np.array([sum(dout[0, 0, i] / (i + 1) for i in range(j, 7)) for j in range(7)])
    assert np.allclose(dv[0, 0], want, rtol=1e-14, atol=1e-14)


def test_gradient_catches_a_dropped_normaliser_term():
    # planted mistake, in a copy on the CPU: leave out d(den) and the finite
    # differences of the definition disagree
    r = _rng(5)
    q, k, v = (r.standard_normal((1, 1, 5, 3)) for _ in range(3))
    dout = r.standard_normal((1, 1, 5, 3))
    P = 4
    s = (q[0, 0] @ k[0, 0].T) / math.sqrt(3)
    mask = np.tril(np.ones((5, 5), dtype=bool))
    T = np.where(mask, oracle.taylor_kernel(s, P), 0.0)
    den = T.sum(1)
    wrong_dv = T.T @ (dout[0, 0] / den[:, None])  # dv is right without the den term
    wrong_dq = ((np.where(mask, (dout[0, 0] / den[:, None]) @ v[0, 0].T, 0.0)
                 * np.where(mask, oracle.taylor_kernel(s, P - 1), 0.0)) @ k[0, 0]) / math.sqrt(3)
    dq, _, dv = oracle.attention_grad(q, k, v, dout, P)
    assert np.allclose(dv[0, 0], wrong_dv, rtol=1e-12)
    assert not np.allclose(dq[0, 0], wrong_dq, rtol=1e-3)
