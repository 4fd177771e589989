"""The cubic behind the sparse kernel's FMA-pipe exponential (``exp2_fma2`` in
``csrc/vsa_device.cuh``), and a float32 model of that routine.

The kernel evaluates 2^x for part of the softmax probabilities on the FMA
pipe instead of the special-function unit:

* clamp x below at -120 (2^-120 is negligible next to the row maximum's 1);
* j = round-to-nearest-even(x), taken by adding and subtracting 1.5 * 2^23;
  f = x - j lies in [-1/2, 1/2];
* 2^f ~= p(f) = c0 + f (c1 + f (c2 + f c3)), three fused multiply-adds;
* 2^x = p(f) * 2^j, the scaling done by adding j to the exponent field.

The coefficients minimise the largest RELATIVE error of p against 2^f on
[-1/2, 1/2] (minimax, found with the Remez exchange algorithm below, all in
float64), then are rounded to float32.  Running this module prints them in the
hex-float form the header uses:

    python -m block_sparse_attention_15_b200.exp2_fit
"""
from __future__ import annotations

import numpy as np

LO, HI = -0.5, 0.5
DEGREE = 3
CLAMP = -120.0
ROUND_MAGIC = np.float32(12582912.0)  # 1.5 * 2^23


def _solve_reference(xs: np.ndarray) -> tuple[np.ndarray, float]:
    """Polynomial c (low order first) and level E with
    p(x_i) = 2^x_i (1 + (-1)^i E) at the DEGREE + 2 reference points."""
    n = DEGREE + 2
    y = np.exp2(xs)
    A = np.zeros((n, n))
    for i in range(n):
        A[i, :DEGREE + 1] = xs[i] ** np.arange(DEGREE + 1)
        A[i, DEGREE + 1] = -((-1.0) ** i) * y[i]
    sol = np.linalg.solve(A, y)
    return sol[:DEGREE + 1], float(sol[DEGREE + 1])


def rel_error(c: np.ndarray, x: np.ndarray) -> np.ndarray:
    return np.polyval(c[::-1], x) / np.exp2(x) - 1.0


def remez(iters: int = 40, grid: int = 200001) -> np.ndarray:
    """Minimax (relative error) polynomial of degree DEGREE for 2^f on
    [LO, HI], float64 coefficients, low order first."""
    # start from the Chebyshev extrema, which are near-optimal already
    k = np.arange(DEGREE + 2)
    xs = 0.5 * (LO + HI) + 0.5 * (HI - LO) * np.cos(np.pi * k[::-1] / (DEGREE + 1))
    fine = np.linspace(LO, HI, grid)
    c = None
    for _ in range(iters):
        c, _ = _solve_reference(xs)
        e = rel_error(c, fine)
        # new reference: the extremum of each sign run of the error
        s = np.sign(e)
        s[s == 0] = 1
        cuts = np.flatnonzero(np.diff(s)) + 1
        runs = np.split(np.arange(grid), cuts)
        ext = np.array([r[np.argmax(np.abs(e[r]))] for r in runs])
        if len(ext) < DEGREE + 2:
            break
        # keep DEGREE + 2 alternating extrema, the largest window of them
        if len(ext) > DEGREE + 2:
            best = max(range(len(ext) - DEGREE - 1),
                       key=lambda i: np.abs(e[ext[i:i + DEGREE + 2]]).min())
            ext = ext[best:best + DEGREE + 2]
        new = fine[ext]
        if np.allclose(new, xs, atol=1e-12, rtol=0):
            break
        xs = new
    return c


def coefficients_f32() -> np.ndarray:
    """The fitted coefficients rounded to float32, low order first."""
    return remez().astype(np.float32)


def _fma32(a, b, c):
    """float32 fused multiply-add modelled in float64: the float32 product is
    exact in float64, the sum is rounded once in float64 and then to float32
    (a double rounding that can differ from a true fused operation by at most
    one float32 ulp, far below the error bounds checked with this model)."""
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def exp2_model(x: np.ndarray, c: np.ndarray | None = None) -> np.ndarray:
    """float32 model of the kernel's steps for 2^x (see the module text)."""
    if c is None:
        c = coefficients_f32()
    c = np.asarray(c, dtype=np.float32)
    x = np.asarray(x, dtype=np.float32)
    xx = np.maximum(x, np.float32(CLAMP))
    t = (xx + ROUND_MAGIC).astype(np.float32)
    j = (t - ROUND_MAGIC).astype(np.float32)
    f = _fma32(j, np.float32(-1.0), xx)
    q = _fma32(f, c[3], c[2])
    q = _fma32(q, f, c[1])
    q = _fma32(q, f, c[0])
    # j added to the exponent field: q * 2^j exactly (no overflow or
    # underflow for x in [-120, 32])
    return (q.astype(np.float64) * np.exp2(j.astype(np.float64))).astype(np.float32)


def hex_literals(c=None) -> list[str]:
    """C99 hex-float literals of the float32 coefficients, low order first."""
    if c is None:
        c = coefficients_f32()
    out = []
    for v in np.asarray(c, dtype=np.float32):
        m, e = np.frexp(np.float64(v))       # v = m * 2^e, 0.5 <= |m| < 1
        mant = int(round(abs(m) * 2 ** 24))  # 24 significant bits
        # print as 0x1.hhhhhhp(e-1): 1 + 23 fraction bits, padded to 24
        frac = (mant - 2 ** 23) << 1
        out.append(f"{'-' if v < 0 else ''}0x1.{frac:06x}p{e - 1}f")
    return out


if __name__ == "__main__":
    c = coefficients_f32()
    xs = np.linspace(LO, HI, 400001)
    print("c0..c3:", ", ".join(hex_literals(c)))
    print("max relative error of the float32 coefficients on [-1/2, 1/2]: "
          f"{np.abs(rel_error(c.astype(np.float64), xs)).max():.3e}")
