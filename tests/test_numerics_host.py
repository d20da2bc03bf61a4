"""Host checks of the kernels' float32 formulas (no GPU): the numerics a kernel relies on,
restated in numpy float32 and compared with fp64 references."""
import numpy as np


def test_zoh_coefficient_formula_in_float32():
    """The kernels' float32 evaluation of the zero-order-hold coefficient (a - 1)/A, with the
    series Δ (1 + x/2 + x²/6 + x³/24 + x⁴/120) for |x| = |ΔA| < 1/4, stays within 2e-6 of
    expm1(ΔA)/A in fp64 over steps and decays spanning the workloads and beyond (the MUFU
    exponential is stood in for by a float32 exp2 perturbed by 2 ulp)."""
    f = np.float32
    dt = np.exp(np.linspace(np.log(1e-4), np.log(8.0), 400)).astype(f)
    A = -np.exp(np.linspace(np.log(1e-3), np.log(60.0), 300)).astype(f)
    Dt, Aa = np.meshgrid(dt, A)
    x2 = (Dt * (Aa * f(np.log2(np.e)))).astype(f)                # Δ·A·log2e as the kernel forms it
    a = np.exp2(x2).astype(f)
    a = (a * f(1 + 2 * 2.0 ** -23)).astype(f)                      # 2 ulp of MUFU error
    x = (x2 * f(np.log(2.0))).astype(f)
    s = (x * f(1 / 120) + f(1 / 24)).astype(f)
    for c in (1 / 6, 0.5, 1.0):
        s = (x * s + f(c)).astype(f)
    near = (Dt * s).astype(f)
    far = ((a - f(1)) * (f(1) / Aa)).astype(f)
    coef = np.where(np.abs(x) < f(0.25), near, far)
    exact = np.expm1(Dt.astype(np.float64) * Aa.astype(np.float64)) / Aa.astype(np.float64)
    rel = np.abs(coef - exact) / np.abs(exact)
    assert rel.max() < 2e-6, rel.max()
    assert np.abs(x).max() > 100 and np.abs(x).min() < 1e-6   # both branches and their far ends


def test_fast_softplus_formula_in_float32():
    """The one-MUFU softplus: w = e^-|x| through ex2, log1p(w) = w q(w) with q a degree-7
    polynomial in w (Horner, float32), plus max(x, 0).  Restated in float32 (the MUFU ex2 stood
    in for by a float32 exp2 perturbed by 2 ulp), it stays within 5e-6 relative of fp64
    softplus over the deltas and biases of the workloads and beyond (the largest errors, ~2e-6
    near |x| = 30, come from rounding |x| log2(e) to float32 before the exponential), far
    inside the 3e-3 bf16 and 1e-4 float32 budgets.  On [-1, 1], where nothing is lost to that
    rounding, it is within 6e-7."""
    f = np.float32
    coef = [0.9999998211860657, -0.4999740421772003, 0.33275479078292847, -0.24495449662208557,
            0.17745204269886017, -0.10768117010593414, 0.044089239090681076, -0.00853909645229578]
    ulp2 = f(1 + 2 * 2.0 ** -23)

    def fast(xs):
        w = (np.exp2((-np.abs(xs)) * f(np.log2(np.e))) * ulp2).astype(f)
        q = f(coef[-1])
        for c in coef[-2::-1]:
            q = (w * q + f(c)).astype(f)
        return (w * q + np.maximum(xs, f(0))).astype(f)

    xs = np.linspace(-30.0, 30.0, 200001).astype(f)
    ref = np.logaddexp(0.0, xs.astype(np.float64))
    assert (np.abs(fast(xs) - ref) / ref).max() < 5e-6
    xs = np.linspace(-1.0, 1.0, 20001).astype(f)
    ref = np.logaddexp(0.0, xs.astype(np.float64))
    assert (np.abs(fast(xs) - ref) / ref).max() < 6e-7
    # the extremes: far below zero the result flushes to (almost) 0, far above it is x
    assert fast(np.array([-200.0], dtype=f))[0] < 1e-30
    assert fast(np.array([200.0], dtype=f))[0] == f(200.0)


def test_fast_silu_formula_in_float32():
    """The 16-bit-input gate silu(z) = z/2 (1 + tanh(z/2)): with a tanh carrying a relative
    error of 2^-11 (the documented bound of the approximate MUFU tanh; about 1e-5 measured),
    the gate stays within 1e-3 of z sigmoid(z) relative to |z|, inside the 3e-3 bf16 budget."""
    f = np.float32
    z = np.linspace(-40.0, 40.0, 100001).astype(f)
    hz = (f(0.5) * z).astype(f)
    t = (np.tanh(hz) * f(1 + 2.0 ** -11)).astype(f)
    got = (hz * t + hz).astype(f)
    ref = z.astype(np.float64) / (1.0 + np.exp(-z.astype(np.float64)))
    assert (np.abs(got - ref) / np.maximum(np.abs(z), 1e-30)).max() < 1e-3
