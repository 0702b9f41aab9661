"""Fits the degree-5 polynomial p(f) ~ 2^f on [-1/2, 1/2] used by the scan's
FMA-pipe exponential, minimising the maximum relative error (Lawson's iteratively
reweighted least squares on a dense grid), and prints the float32 coefficients.
The constant term is pinned to 1 (p(f) = 1 + f q(f)) so that p(0) = 1
exactly: decays close to 1 then carry an error proportional to |f| instead of
a fixed offset, which a long memory 1 / (1 - dA) would amplify.

    python -m selective_state_space_08_b200.csrc.gen_exp2_poly

The kernel evaluates 2^x = 2^j * p(x - j) with j = rint(x) (Cody-Waite style
range reduction); the coefficients below are pasted into exp2_poly.cuh.
"""
import numpy as np

DEG = 5
LO, HI = -0.5, 0.5


def fit(deg=DEG, iters=400):
    """Lawson's algorithm (iteratively reweighted least squares) for the
    minimax relative error with the constant term fixed at 1."""
    grid = np.linspace(LO, HI, 4001)
    target = 2.0 ** grid
    # relative error of 1 + sum_j c_j f^j:  (sum_j c_j f^j - (2^f - 1)) / 2^f
    V = np.stack([grid ** j for j in range(1, deg + 1)], axis=1) / target[:, None]
    rhs = (target - 1.0) / target
    w = np.full(grid.size, 1.0 / grid.size)
    for _ in range(iters):
        sw = np.sqrt(w)
        c, *_ = np.linalg.lstsq(V * sw[:, None], rhs * sw, rcond=None)
        err = np.abs(V @ c - rhs)
        w = w * err
        w /= w.sum()
    c = np.concatenate([[1.0], c])
    return c, float(np.max(np.abs(V @ c[1:] - rhs)))


def main():
    c, e = fit()
    c32 = c.astype(np.float32)
    grid = np.linspace(LO, HI, 100001).astype(np.float32)
    p = np.zeros_like(grid)
    for cj in c32[::-1]:
        p = (p * grid + cj).astype(np.float32)
    rel = np.max(np.abs(p.astype(np.float64) - 2.0 ** grid.astype(np.float64)) / 2.0 ** grid)
    print(f"// max relative error: minimax {e:.3e}, float32 Horner {rel:.3e}")
    for j, cj in enumerate(c32):
        print(f"constexpr float kExp2C{j} = {float(cj):.9e}f;")


if __name__ == "__main__":
    main()
