"""Where the weight-gradient tolerance of the GPU backward tests comes from.

The backward of the grouped SwiGLU rounds its intermediates the way the
kernels store them: G = S w1^T and U = S w3^T rounded once to bf16 (kept by
the training forward), H = silu(G) U rounded to bf16, dG and dU rounded to
bf16 before the next products, every output rounded once to bf16; all
products accumulate in fp32.  This module replays exactly those roundings
in fp64 (the fp32 accumulation itself is left exact: its error is orders
of magnitude below one bf16 rounding) on the segment mixes the GPU tests
use, and compares the result with the oracle's exact chain rule
(oracle.grouped_swiglu_backward, no intermediate rounding).

The tolerances the GPU tests apply to the weight gradients, per expert,
  max|err| <= 6e-2 (|ref| + rms(ref))  and  ||err||_F <= 1e-2 ||ref||_F,
must hold with a factor of two to spare for this emulated error alone: the
rest of the margin covers fp32 accumulation order and the fast exponential
of the kernels' SiLU.  If a change to the rounding chain (or to the oracle)
pushed the emulated error past half the tolerance, this test fails.
"""
import numpy as np
import pytest
import torch

import oracle as O
from test_gpu_backward import CASES, expert_problem

# the tolerances of tests/test_gpu_backward.py (close_wgrad and close)
WGRAD_MAX, WGRAD_FRO = 6e-2, 1e-2
BF16_MAX, BF16_FRO = 3e-2, 1e-2


def rb(a):
    """fp64 -> the fp32 value a kernel holds -> one RNE rounding to bf16."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float64)).to(torch.float32)
    return t.to(torch.bfloat16).to(torch.float64).numpy()


def emulated_backward(xp, off, w1, w3, w2, dy):
    """The kernels' rounding chain, one expert segment at a time."""
    S_all, g_all = O.as_f64(xp), O.as_f64(dy)
    E = len(off) - 1
    h, d = w1.shape[1], w1.shape[2]
    dxp = np.zeros_like(S_all)
    dw1, dw3, dw2 = np.zeros((E, h, d)), np.zeros((E, h, d)), np.zeros((E, d, h))
    for e in range(E):
        lo, hi = int(off[e]), int(off[e + 1])
        if hi == lo:
            continue
        S, dY = S_all[lo:hi], g_all[lo:hi]
        W1, W3, W2 = O.as_f64(w1[e]), O.as_f64(w3[e]), O.as_f64(w2[e])
        G, U = S @ W1.T, S @ W3.T
        Gb, Ub = rb(G), rb(U)                     # kept by the training forward
        Hb = rb(O.silu(G) * U)                    # forward epilogue, from fp32 G, U
        dA = dY @ W2
        dU = rb(dA * O.silu(Gb))                  # SwiGLU' epilogue reads the bf16 G, U
        dG = rb(dA * Ub * O.silu_grad(Gb))
        dxp[lo:hi] = rb(dG @ W1 + dU @ W3)
        dw2[e] = rb(dY.T @ Hb)
        dw1[e] = rb(dG.T @ S)
        dw3[e] = rb(dU.T @ S)
    return dxp, dw1, dw3, dw2


def wgrad_errors(got, ref):
    rms = np.sqrt(np.mean(ref ** 2))
    err = np.abs(got - ref)
    return (err / (np.abs(ref) + rms)).max(), np.linalg.norm(got - ref) / np.linalg.norm(ref)


@pytest.mark.parametrize("counts,d,h", CASES)
def test_weight_gradient_tolerance_covers_the_rounding_chain(counts, d, h):
    # the same inputs as test_grouped_swiglu_backward_matches_oracle
    xp, w1, w3, w2, dy, off = expert_problem(counts, d, h, seed=7 * sum(counts) + h)
    rdx, rw1, rw3, rw2 = O.grouped_swiglu_backward(xp, off, w1, w3, w2, dy)
    edx, ew1, ew3, ew2 = emulated_backward(xp, off, w1, w3, w2, dy)
    worst_max, worst_fro = 0.0, 0.0
    for e, n in enumerate(counts):
        if n == 0:
            assert not ew1[e].any() and not ew3[e].any() and not ew2[e].any()
            continue
        for got, ref in ((ew1[e], rw1[e]), (ew3[e], rw3[e]), (ew2[e], rw2[e])):
            m, f = wgrad_errors(got, ref)
            worst_max, worst_fro = max(worst_max, m), max(worst_fro, f)
    print(f"counts={counts} d={d} h={h}: emulated weight-gradient error "
          f"max err/(|ref|+rms) = {worst_max:.4f}, Frobenius {worst_fro:.4%}")
    assert worst_max <= WGRAD_MAX / 2, worst_max
    assert worst_fro <= WGRAD_FRO / 2, worst_fro
    # the data gradient meets the plain bf16 tolerance with the same margin
    err = np.abs(edx - rdx)
    assert (err / (1 + np.abs(rdx))).max() <= BF16_MAX / 2
    assert np.linalg.norm(edx - rdx) <= BF16_FRO / 2 * np.linalg.norm(rdx)


def test_rounding_chain_is_what_makes_the_error():
    """The emulation without any intermediate rounding is the oracle (to
    fp64 rounding): the error measured above comes from the bf16 chain."""
    counts, d, h = CASES[1]
    xp, w1, w3, w2, dy, off = expert_problem(counts, d, h, seed=3)
    _, rw1, rw3, rw2 = O.grouped_swiglu_backward(xp, off, w1, w3, w2, dy)
    global rb
    saved = rb
    try:
        rb = lambda a: np.asarray(a, dtype=np.float64)  # noqa: E731
        _, ew1, ew3, ew2 = emulated_backward(xp, off, w1, w3, w2, dy)
    finally:
        rb = saved
    for got, ref in ((ew1, rw1), (ew3, rw3), (ew2, rw2)):
        assert np.allclose(got, ref, rtol=1e-12, atol=1e-12)
