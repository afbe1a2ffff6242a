"""Float64 CPU oracle for alpha-entmax attention (AdaSplash / AdaSplash-2).

TEST INFRASTRUCTURE ONLY. Only the tests, the smoke check in
`__graft_entry__.smoke()` and the CPU-baseline leg of `bench.py` may import
this package. The product path (the CUDA library and its Python binding)
never calls it, and it shares no code with that path.

What it computes, in plain float64 numpy:

* `entmax.tau_bisect`: the normaliser tau of alpha-entmax,
  p_j = [z_j - tau]_+^{1/(alpha-1)} with sum_j p_j = 1, found by bisection
  to 1e-12 (AdaSplash-2 summary, gist.science (de), section 1
  "Problemstellung": tau needs an iterative root search).
* `entmax.histogram_tau`: the left-edge histogram lower bound tau_h
  (AdaSplash-2 summary, gist.science (de), section 2, "Streaming &
  Histogramm-Erstellung" and "Theoretische Garantie").
* `entmax.hybrid_solve`: the safeguarded Halley / Newton / secant solver
  with bisection fallback, started from tau_h (same page, "Hybrid Solver &
  Sparsity-Awareness"; AdaSplash-2 technical summary, gist.science (hi),
  section 2, hybrid solver strategy).
* `softmax.forward` / `softmax.backward`: dense softmax attention, the
  reference for the in-library dense baseline.
* `attention.forward` / `attention.backward`: entmax attention
  O = P V with s = Q K^T / sqrt(d), z = (alpha - 1) s, the bit-packed block
  mask (32 blocks per 32-bit word; gist.science (de), "Bit-Packed Block
  Mask"), and the analytic gradient dS = u * (g - delta),
  u = p^{2 - alpha}, delta = sum(u g) / sum(u).

Parity pins: every function is pinned by `tests/test_oracle_pins.py`
against closed forms, brute force and finite differences; none is
"parity unpinned".
"""

from . import entmax, attention, softmax  # noqa: F401
