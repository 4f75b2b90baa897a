"""Coefficients of the polynomial behind the forward kernel's FMA-pipe 2^x.

The forward kernel computes some of its exponentials without the MUFU unit: with
x = i + f, i = round(x) and f in [-1/2, 1/2] (the Cody-Waite style argument split of
W. J. Cody and W. Waite, "Software Manual for the Elementary Functions", 1980),
2^x = 2^i * 2^f, where 2^i goes into the exponent field and 2^f comes from a
polynomial c0 + c1 f + ... + cn f^n. This module fits that polynomial: the minimax
approximation of 2^f on [-1/2, 1/2] in RELATIVE error, by the Remez exchange
algorithm (E. Ya. Remez, 1934) on a dense grid, in float64. The coefficients are then
rounded to float32, the precision the kernel holds them in.

`python -m exact_io_aware_69_b200.fit_exp2` prints them in the form that
csrc/sm100.cuh spells out; tests check that the two agree and that the float32
evaluation stays within the stated bound.
"""
from __future__ import annotations

import numpy as np

DEGREE = 4
LO, HI = -0.5, 0.5


def _solve_levelled(nodes: np.ndarray, degree: int) -> tuple[np.ndarray, float]:
    """Coefficients c and level E with (p(x_k) - 2^x_k) / 2^x_k = (-1)^k E at the n+2 nodes."""
    n = degree + 1
    a = np.zeros((n + 1, n + 1))
    for k, x in enumerate(nodes):
        a[k, :n] = x ** np.arange(n)
        a[k, n] = -((-1.0) ** k) * 2.0 ** x
    coef = np.linalg.solve(a, 2.0 ** nodes)
    return coef[:n], coef[n]


def fit(degree: int = DEGREE, grid: int = 200001, iters: int = 30) -> np.ndarray:
    """Minimax (relative error) polynomial for 2^f on [LO, HI], lowest power first."""
    xs = np.linspace(LO, HI, grid)
    k = np.arange(degree + 2)
    nodes = 0.5 * (LO + HI) - 0.5 * (HI - LO) * np.cos(np.pi * k / (degree + 1))  # Chebyshev
    c = None
    for _ in range(iters):
        c, _ = _solve_levelled(nodes, degree)
        err = np.polyval(c[::-1], xs) / 2.0 ** xs - 1.0
        # new nodes: the extremum of the error on each interval of constant sign
        sign_change = np.nonzero(np.diff(np.sign(err)))[0]
        bounds = np.concatenate(([0], sign_change + 1, [grid]))
        ext = [b0 + int(np.argmax(np.abs(err[b0:b1]))) for b0, b1 in zip(bounds[:-1], bounds[1:])]
        if len(ext) != degree + 2:
            break
        new = xs[ext]
        if np.allclose(new, nodes, rtol=0, atol=1e-12):
            break
        nodes = new
    return c


def coefficients() -> list[float]:
    """The fitted coefficients rounded to float32 (lowest power first)."""
    return [float(np.float32(v)) for v in fit()]


def eval_f32(x: np.ndarray, coef: list[float] | None = None) -> np.ndarray:
    """The kernel's steps in float32: clamp, split by the 1.5 * 2^23 shifter, Horner,
    exponent add (fused multiply-adds emulated by rounding the float64 result once)."""
    coef = coefficients() if coef is None else coef
    c = [np.float32(v) for v in coef]
    x = np.maximum(np.asarray(x, np.float32), np.float32(-125.0))
    shifter = np.float32(12582912.0)
    t = (x + shifter).astype(np.float32)
    f = (x - (t - shifter).astype(np.float32)).astype(np.float32)
    p = np.full_like(f, c[-1])
    for ck in c[-2::-1]:
        p = (p.astype(np.float64) * f.astype(np.float64) + np.float64(ck)).astype(np.float32)
    bits = p.view(np.int32).astype(np.int64) + (t.view(np.int32).astype(np.int64) << 23)
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


def max_rel_error(coef: list[float] | None = None, n: int = 400001) -> float:
    """Largest relative error of eval_f32 against 2^x over x in [-60, 8]."""
    x = np.linspace(-60.0, 8.0, n).astype(np.float32)
    y = eval_f32(x, coef).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    return float(np.max(np.abs(y / ref - 1.0)))


if __name__ == "__main__":
    for k, v in enumerate(coefficients()):
        print(f"c{k} = {v!r}f")
    print(f"max relative error (float32 evaluation): {max_rel_error():.3e}")
