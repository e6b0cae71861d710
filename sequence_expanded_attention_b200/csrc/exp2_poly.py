"""Derivation of the polynomial behind ex2_poly() in hd_ptx.cuh.

The prefill softmax evaluates 2^x for a share of its scores on the FMA pipe
instead of the MUFU unit.  Method (Cody-Waite range reduction):

    x = j + f,  j = round-to-nearest(x),  f in [-1/2, 1/2]
    2^x = 2^j * 2^f,  2^f ~= c0 + c1 f + c2 f^2 + c3 f^3

and 2^j is applied by adding j to the float's exponent field.  The cubic is
fitted here by weighted least squares on Chebyshev nodes, minimising the
relative error (weights 1 / 2^f), which lands close to the minimax cubic.
The result feeds a bf16 probability (8 significant bits, unit roundoff
2^-9 = 1.95e-3), so a relative error near 1e-4 is far below what the
rounding already costs.

    python -m sequence_expanded_attention_b200.csrc.exp2_poly   # prints the constants
"""
import numpy as np

DEGREE = 3


def fit(degree: int = DEGREE, nodes: int = 4096):
    k = np.arange(nodes)
    f = 0.5 * np.cos(np.pi * (k + 0.5) / nodes)  # Chebyshev nodes on [-1/2, 1/2]
    target = np.exp2(f)
    A = np.vander(f, degree + 1, increasing=True) / target[:, None]
    c, *_ = np.linalg.lstsq(A, np.ones_like(f), rcond=None)
    return c


def horner_f32(c, f):
    """Evaluate the cubic the way the kernel does: fp32 Horner with FMA."""
    c = np.asarray(c, dtype=np.float32)
    f = np.asarray(f, dtype=np.float32)
    p = np.full_like(f, c[-1])
    for ci in c[-2::-1]:
        p = (p.astype(np.float64) * f + ci).astype(np.float32)  # one rounding, as an FMA
    return p


def max_rel_error(c, samples: int = 200001):
    f = np.linspace(-0.5, 0.5, samples, dtype=np.float64)
    p = horner_f32(c, f.astype(np.float32)).astype(np.float64)
    return float(np.max(np.abs(p / np.exp2(f) - 1.0)))


if __name__ == "__main__":
    c = fit()
    for i, ci in enumerate(np.asarray(c, dtype=np.float32)):
        print(f"c{i} = {float(ci):.9e}f")
    print(f"max relative error on [-1/2, 1/2] (fp32 Horner): {max_rel_error(c):.3e}")
