"""Fits the polynomial of the FMA-pipe base-2 exponential used by the scoring epilogue.

Method: range reduction x = n + f with n = round-to-nearest(x) and f in [-1/2, 1/2] (the
1.5 * 2^23 shifter trick), 2^f by a polynomial, and 2^n applied by adding n to the exponent
field. The polynomial minimises the maximum RELATIVE error of p(f) against 2^f on [-1/2, 1/2]
(Remez-style exchange on a dense grid, solved as a linear program-free iteration: weighted
least squares with Lawson's multiplicative weight update). Run:

    python decode_kv_cache_kara_b200/csrc/gen_exp2_poly.py [degree]

It prints the coefficients (c0 + c1 f + ... ) as float32 hex and decimal, and the maximum
relative error of the float32 Horner evaluation over the whole reduced range.
"""

import sys

import numpy as np


def fit(degree: int, iters: int = 400):
    f = np.cos(np.linspace(0, np.pi, 20001)) * 0.5          # Chebyshev-clustered grid
    y = np.exp2(f)
    a = np.vander(f, degree + 1, increasing=True) / y[:, None]
    w = np.ones_like(f) / len(f)
    c = None
    for _ in range(iters):                                   # Lawson's algorithm (minimax)
        sw = np.sqrt(w)
        c, *_ = np.linalg.lstsq(a * sw[:, None], sw, rcond=None)
        err = np.abs(a @ c - 1.0)
        w = w * err
        w /= w.sum()
    return c


def horner32(c32, f32):
    r = np.full_like(f32, c32[-1])
    for ci in c32[-2::-1]:
        r = (r * f32 + ci).astype(np.float32)
    return r


def main():
    degree = int(sys.argv[1]) if len(sys.argv) > 1 else 4
    c = fit(degree)
    c32 = c.astype(np.float32)
    x = np.linspace(-126.0, 0.0, 2_000_001).astype(np.float32)
    shifter = np.float32(12582912.0)
    t = (x + shifter).astype(np.float32)
    n = (t - shifter).astype(np.float32)
    f = (x - n).astype(np.float32)
    p = horner32(c32, f)
    bits = p.view(np.int32) + (t.view(np.int32) << 23)
    got = bits.view(np.float32).astype(np.float64)
    rel = np.abs(got / np.exp2(x.astype(np.float64)) - 1.0)
    for i, ci in enumerate(c32):
        print(f"c{i} = {float(ci)!r:>24}  (0x{ci.view(np.uint32):08x})")
    print(f"max relative error over [-126, 0]: {rel.max():.3e}")


if __name__ == "__main__":
    main()
