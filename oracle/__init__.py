"""fp64 CPU oracle for causal SATA (symmetry-aware Taylor approximation) attention.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / reference leg of ``bench.py`` may import this package.  The
CUDA library never calls it and shares no code, table or constant with it; the
only common module is ``sata_inputs`` (random draws, no method arithmetic).

Sources (web pages; cited by title and section):

* [SATA-eng] "对称性感知泰勒近似注意力机制的恒定计算成本工程实现"
  (blog.hotdry.top, symmetry-aware Taylor approximation, constant-cost
  engineering), sections
    - "对称张量分解的核心洞察"   (symmetric-tensor insight: Taylor series of
      exp(q.k), d_K^p monomials of (q^T k)^p, minimal basis of size
      C(d_K+p-1, p) made of the upper-triangular index region, fixed tables M_p),
    - "恒定计算成本的工程实现"   (constant-cost implementation: hidden state of
      (d_V+1) x C(d_K+P-1, P-1) elements, per-token procedure, FLOP formula),
    - "精度与效率的权衡参数"     (precision/efficiency trade-off in P),
    - "硬件优化路径与当前局限"   (index hierarchy i_1 <= i_2 <= ... <= i_p).
* [Attn-var] "Transformer 注意力机制变体与长序列建模优化：从 O(n²) 到线性注意力的工程演进"
  (mokono.cn), section "2.1 标准注意力实现与瓶颈分析": layout
  (batch, heads, seq_len, dim) and score scale dim**-0.5.
* [SATA-faq] "对称感知泰勒近似实现恒定Token成本注意力机制" (ai-stack.site),
  FAQ 5 (models trained from scratch with the method: the reason for a
  backward pass).

Readings where the pages are silent:
degrees 0..P-1; inclusive causal mask j <= i; one normaliser shared by all
degrees; no eps, clamp or max-subtraction; weights 1/sqrt(alpha! d_K^(p/2))
(square root of the multinomial count times the Taylor 1/p! and the score
scale, split evenly between the query and the key side).

Modules: ``basis`` (M_p tables and weights), ``sata`` (quadratic form,
feature-map form, decode step, exact softmax, cost formulas), ``brute``
(full d_K^p ordered-tuple expansion for tiny d_K).
"""
from .basis import basis_rows, basis_weights, basis_all, multiplicity_factorial
from .sata import (
    taylor_kernel,
    feature_map,
    quadratic_form,
    attention_grad,
    conditioning,
    feature_form,
    decode_step,
    final_state,
    softmax_attention,
    basis_total,
    flops_per_token_counted,
)

__all__ = [
    "basis_rows", "basis_weights", "basis_all", "multiplicity_factorial",
    "taylor_kernel", "feature_map", "quadratic_form", "attention_grad", "conditioning",
    "feature_form",
    "decode_step", "final_state", "softmax_attention", "basis_total",
    "flops_per_token_counted",
]
