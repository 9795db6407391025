"""fp64 CPU reference computations for causal SATA attention (test infrastructure only).

Definition followed (per head; s_ij = q_i.k_j / sqrt(d_K), the dim**-0.5 scale of
[Attn-var] section "2.1 标准注意力实现与瓶颈分析"):

    T_P(s)  = sum_{p=0}^{P-1} s^p / p!        (exp(s) truncated; [SATA-eng]
                                                 "对称张量分解的核心洞察")
    num_i   = sum_{j<=i} T_P(s_ij) v_j
    den_i   = sum_{j<=i} T_P(s_ij)
    out_i   = num_i / den_i

[SATA-eng] states that the symmetric reorganisation leaves attention's
definition unchanged; so the quadratic form above and the feature-map form
(per-token update of a fixed-size state, section "恒定计算成本的工程实现") must
agree up to rounding.  All arithmetic is float64 from the exact input values.
[SATA-faq] is "对称感知泰勒近似实现恒定Token成本注意力机制" (ai-stack.site), whose
FAQ 5 reports models trained from scratch with the method (attention_grad).
"""
from __future__ import annotations

import math

import numpy as np

from .basis import basis_all, basis_rows


def _f64(x) -> np.ndarray:
    if hasattr(x, "detach"):  # torch tensor: exact widening of fp32/bf16 values
        import torch

        return x.detach().cpu().to(torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def taylor_kernel(s, P: int) -> np.ndarray:
    """T_P(s) = sum of s^p / p! for p = 0..P-1, as a plain sum of powers."""
    s = np.asarray(s, dtype=np.float64)
    total = np.zeros_like(s)
    for p in range(P):
        total = total + s ** p / math.factorial(p)
    return total


def basis_total(dK: int, P: int) -> int:
    """m = number of rows of M_0 .. M_{P-1} together (by enumeration)."""
    return int(sum(len(basis_rows(dK, p)) for p in range(P)))


def feature_map(x, P: int, basis=None) -> np.ndarray:
    """phi(x) for x [..., dK]: for each degree p and each row alpha of M_p,
    w_alpha * prod_r x[alpha_r]; degrees concatenated p = 0..P-1 -> [..., m]."""
    x = _f64(x)
    dK = x.shape[-1]
    if basis is None:
        basis = basis_all(dK, P)
    parts = []
    for p, rows, w in basis:
        if p == 0:
            mono = np.ones(x.shape[:-1] + (1,), dtype=np.float64)
        else:
            mono = np.prod(x[..., rows], axis=-1)  # [..., count]
        parts.append(mono * w)
    return np.concatenate(parts, axis=-1)


def _heads(q, k, v):
    q, k, v = _f64(q), _f64(k), _f64(v)
    if q.ndim != 4 or k.shape != q.shape or v.shape[:3] != q.shape[:3]:
        raise ValueError("expected q,k [B,H,N,dK] and v [B,H,N,dV]")
    return q, k, v


def quadratic_form(q, k, v, P: int, row_block: int = 1024):
    """Form (a): the definition written out, O(N^2) per head.

    Returns (num [B,H,N,dV], den [B,H,N], out [B,H,N,dV]).  Rows are evaluated in
    groups of ``row_block`` only to bound memory; each row's arithmetic is the
    definition: scores, causal mask j <= i, T_P, weighted sums.
    """
    q, k, v = _heads(q, k, v)
    B, H, N, dK = q.shape
    dV = v.shape[-1]
    scale = 1.0 / math.sqrt(dK)
    num = np.zeros((B, H, N, dV))
    den = np.zeros((B, H, N))
    for b in range(B):
        for h in range(H):
            for i0 in range(0, N, row_block):
                i1 = min(N, i0 + row_block)
                s = (q[b, h, i0:i1] @ k[b, h, :i1].T) * scale          # [rows, i1]
                t = taylor_kernel(s, P)
                mask = np.arange(i1)[None, :] <= np.arange(i0, i1)[:, None]
                t = np.where(mask, t, 0.0)
                num[b, h, i0:i1] = t @ v[b, h, :i1]
                den[b, h, i0:i1] = t.sum(axis=1)
    return num, den, num / den[..., None]


def attention_grad(q, k, v, dout, P: int):
    """Gradients of L = sum(dout * out) with respect to q, k, v, where out is
    the definition above: the backward pass a training step needs ([SATA-faq],
    FAQ 5, on training models with the method from scratch).  Chain rule through the
    definition, per head, with T = T_P(s) and s = q k^T / sqrt(d_K) on j <= i:

        dnum_i = dout_i / den_i
        dden_i = -(dout_i . out_i) / den_i
        dT_ij  = dnum_i . v_j + dden_i
        dv_j   = sum_{i >= j} T_ij dnum_i
        ds_ij  = dT_ij * T_{P-1}(s_ij)        (d/ds of sum_{p<P} s^p/p!)
        dq_i   = sum_{j <= i} ds_ij k_j / sqrt(d_K)
        dk_j   = sum_{i >= j} ds_ij q_i / sqrt(d_K)

    Returns (dq, dk, dv) with the shapes of q, k, v.  O(N^2) per head.
    """
    q, k, v = _heads(q, k, v)
    dout = _f64(dout)
    B, H, N, dK = q.shape
    scale = 1.0 / math.sqrt(dK)
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    mask = np.arange(N)[None, :] <= np.arange(N)[:, None]
    for b in range(B):
        for h in range(H):
            s = (q[b, h] @ k[b, h].T) * scale
            T = np.where(mask, taylor_kernel(s, P), 0.0)
            Td = np.where(mask, taylor_kernel(s, P - 1), 0.0)
            num = T @ v[b, h]
            den = T.sum(axis=1)
            out = num / den[:, None]
            dnum = dout[b, h] / den[:, None]
            dden = -(dout[b, h] * out).sum(axis=1) / den
            dT = np.where(mask, dnum @ v[b, h].T + dden[:, None], 0.0)
            dv[b, h] = T.T @ dnum
            ds = dT * Td
            dq[b, h] = (ds @ k[b, h]) * scale
            dk[b, h] = (ds.T @ q[b, h]) * scale
    return dq, dk, dv


def conditioning(q, k, P: int, row_block: int = 1024) -> np.ndarray:
    """sum_{j<=i} |T_P(s_ij)| per row [B,H,N]: the scale against which rounding
    in den_i = sum_{j<=i} T_P(s_ij) is measured (T_P is negative for some s
    when P is even, so den_i can be much smaller than this sum)."""
    q, k = _f64(q), _f64(k)
    B, H, N, dK = q.shape
    scale = 1.0 / math.sqrt(dK)
    out = np.zeros((B, H, N))
    for b in range(B):
        for h in range(H):
            for i0 in range(0, N, row_block):
                i1 = min(N, i0 + row_block)
                s = (q[b, h, i0:i1] @ k[b, h, :i1].T) * scale
                t = np.abs(taylor_kernel(s, P))
                mask = np.arange(i1)[None, :] <= np.arange(i0, i1)[:, None]
                out[b, h, i0:i1] = np.where(mask, t, 0.0).sum(axis=1)
    return out


def feature_form(q, k, v, P: int, state0=None):
    """Form (b): the per-token procedure of [SATA-eng] "恒定计算成本的工程实现".

    For each token t in order: map k_t through M_p to phi(k_t), add
    phi(k_t) [v_t, 1]^T to the state S (m x (dV+1), last column = normaliser),
    then read [num_t, den_t] = phi(q_t)^T S.  Returns (num, den, out, S) with S
    the state after the last token, shape [B,H,m,dV+1].
    """
    q, k, v = _heads(q, k, v)
    B, H, N, dK = q.shape
    dV = v.shape[-1]
    basis = basis_all(dK, P)
    m = sum(len(rows) for _, rows, _ in basis)
    num = np.zeros((B, H, N, dV))
    den = np.zeros((B, H, N))
    S_out = np.zeros((B, H, m, dV + 1))
    for b in range(B):
        for h in range(H):
            S = np.zeros((m, dV + 1)) if state0 is None else _f64(state0)[b, h].copy()
            fq = feature_map(q[b, h], P, basis)  # [N, m]
            fk = feature_map(k[b, h], P, basis)
            for t in range(N):
                vt1 = np.append(v[b, h, t], 1.0)
                S += np.outer(fk[t], vt1)
                y = fq[t] @ S
                num[b, h, t] = y[:dV]
                den[b, h, t] = y[dV]
            S_out[b, h] = S
    return num, den, num / den[..., None], S_out


def decode_step(q, k, v, state, P: int):
    """One single-token step on an existing state (update, then read).

    q, k [B,H,dK], v [B,H,dV], state [B,H,m,dV+1] -> (out [B,H,dV], new state).
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    S = _f64(state).copy()
    dV = v.shape[-1]
    fq = feature_map(q, P)
    fk = feature_map(k, P)
    v1 = np.concatenate([v, np.ones(v.shape[:-1] + (1,))], axis=-1)
    S += fk[..., :, None] * v1[..., None, :]
    y = np.einsum("bhm,bhmc->bhc", fq, S)
    return y[..., :dV] / y[..., dV:], S


def final_state(k, v, P: int, token_block: int = 1024):
    """S after N tokens = sum_j phi(k_j) [v_j, 1]^T, with the token sum taken by
    matrix products over blocks of tokens.  [B,H,m,dV+1]."""
    k, v = _f64(k), _f64(v)
    B, H, N, dK = k.shape
    dV = v.shape[-1]
    basis = basis_all(dK, P)
    m = sum(len(rows) for _, rows, _ in basis)
    S = np.zeros((B, H, m, dV + 1))
    for b in range(B):
        for h in range(H):
            for t0 in range(0, N, token_block):
                t1 = min(N, t0 + token_block)
                fk = feature_map(k[b, h, t0:t1], P, basis)
                v1 = np.concatenate([v[b, h, t0:t1], np.ones((t1 - t0, 1))], axis=1)
                S[b, h] += fk.T @ v1
    return S


def softmax_attention(q, k, v, row_block: int = 1024) -> np.ndarray:
    """Exact causal softmax attention with the same scale (max-subtracted exp)."""
    q, k, v = _heads(q, k, v)
    B, H, N, dK = q.shape
    out = np.zeros(v.shape)
    scale = 1.0 / math.sqrt(dK)
    for b in range(B):
        for h in range(H):
            for i0 in range(0, N, row_block):
                i1 = min(N, i0 + row_block)
                s = (q[b, h, i0:i1] @ k[b, h, :i1].T) * scale
                mask = np.arange(i1)[None, :] <= np.arange(i0, i1)[:, None]
                s = np.where(mask, s, -np.inf)
                e = np.exp(s - s.max(axis=1, keepdims=True))
                out[b, h, i0:i1] = (e @ v[b, h, :i1]) / e.sum(axis=1, keepdims=True)
    return out


def flops_per_token_counted(dK: int, dV: int, P: int) -> int:
    """Operations per token of the per-token procedure, counted on the tables.

    update and readout: one multiply and one add per state element each, over
    m x (dV+1) elements; features: a degree-p row costs p multiplies (p-1
    index products and the weight) for q and again for k.
    """
    m = 0
    feat = 0
    for p in range(P):
        cnt = len(basis_rows(dK, p))
        m += cnt
        feat += p * cnt
    return 4 * (dV + 1) * m + 2 * feat
