"""Generator of the cubic in exp2_poly2 (ptx.cuh): the softmax's 2^x on the
FMA pipe evaluates 2^f for f in [-1/2, 1/2] with this polynomial after a
Cody-Waite split x = i + f.

The coefficients are the plain least-squares fit, in fp64, of 2^f at the
n = 2000 Chebyshev nodes f_k = cos((2k + 1) pi / (2n)) / 2 of [-1/2, 1/2],
rounded to float32 where the kernel uses them.

    python fit_exp2_poly.py        # prints the four coefficients c0..c3
"""
import numpy as np

NODES = 2000


def fit(nodes: int = NODES) -> np.ndarray:
    """Coefficients c0..c3 (fp64) of c0 + c1 f + c2 f^2 + c3 f^3 ~ 2^f."""
    k = np.arange(nodes)
    f = 0.5 * np.cos((2 * k + 1) * np.pi / (2 * nodes))
    A = np.vander(f, 4, increasing=True)
    c, *_ = np.linalg.lstsq(A, np.exp2(f), rcond=None)
    return c


if __name__ == "__main__":
    for i, c in enumerate(fit()):
        print(f"c{i} = {float(np.float32(c))!r}")
