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
