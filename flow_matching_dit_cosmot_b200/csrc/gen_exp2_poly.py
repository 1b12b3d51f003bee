"""Coefficients of the degree-3 polynomial p(f) ~ 2^f on [-1/2, 1/2] used by the
attention softmax to compute part of its exponentials on the FMA pipe.

Method: Lawson's algorithm (iteratively reweighted least squares) converging to
the minimax fit of the *relative* error |p(f)/2^f - 1| on a dense grid; the
result is rounded to float32.  Run:

    python flow_matching_dit_cosmot_b200/csrc/gen_exp2_poly.py

and paste the printed constants into attention.cu.  The kernel's own test
(tests/test_gpu_kernels.py, attention parity) and `check()` below bound the
error.
"""

import numpy as np


def fit(degree: int = 3, iters: int = 400):
    f = np.linspace(-0.5, 0.5, 20001)
    y = np.exp2(f)
    V = np.vander(f, degree + 1, increasing=True) / y[:, None]  # relative error
    w = np.ones_like(f) / len(f)
    for _ in range(iters):
        sw = np.sqrt(w)
        c, *_ = np.linalg.lstsq(V * sw[:, None], np.ones_like(f) * sw, rcond=None)
        err = np.abs(V @ c - 1.0)
        w = w * err
        w /= w.sum()
    return c.astype(np.float32)


def check(c):
    f = np.linspace(-0.5, 0.5, 200001).astype(np.float32)
    p = np.zeros_like(f)
    for k in reversed(range(len(c))):
        p = p * f + c[k]
    return float(np.max(np.abs(p.astype(np.float64) / np.exp2(f.astype(np.float64)) - 1.0)))


if __name__ == "__main__":
    c = fit()
    for k, v in enumerate(c):
        print(f"constexpr float kExp2C{k} = {float(v)!r}f;  // 0x{np.float32(v).view(np.uint32):08x}")
    print(f"// max relative error on [-1/2, 1/2]: {check(c):.3e}")
