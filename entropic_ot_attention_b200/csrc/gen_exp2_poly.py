"""Coefficients of the degree-5 polynomial p(f) ~ 2^f on f in [-1/2, 1/2] used by the
FMA-pipe exp2 in tc.cu (Cody-Waite range reduction x = j + f, j = round(x), then
2^x = p(f) * 2^j).  The polynomial interpolates 2^f at the six Chebyshev nodes of the
interval (Chebyshev interpolation: near-minimax); coefficients are rounded to float32 and
the float32 Horner evaluation is checked against the float64 exponential.

    python entropic_ot_attention_b200/csrc/gen_exp2_poly.py
"""
import numpy as np

DEG = 5


def coefficients():
    k = np.arange(DEG + 1)
    nodes = 0.5 * np.cos((2 * k + 1) * np.pi / (2 * (DEG + 1)))
    V = np.vander(nodes, DEG + 1, increasing=True)
    c = np.linalg.solve(V, np.exp2(nodes))
    return c.astype(np.float32)


def max_rel_error(c, n=200001):
    f = np.linspace(-0.5, 0.5, n).astype(np.float32)
    p = np.zeros_like(f)
    for ci in c[::-1]:
        p = (p * f + ci).astype(np.float32)
    ref = np.exp2(f.astype(np.float64))
    return float(np.max(np.abs(p.astype(np.float64) - ref) / ref))


if __name__ == "__main__":
    c = coefficients()
    for i, ci in enumerate(c):
        print(f"c{i} = {float(ci):.9e}f  // {np.float32(ci).view(np.uint32):#010x}")
    print(f"max relative error on [-1/2, 1/2]: {max_rel_error(c):.3e}")
