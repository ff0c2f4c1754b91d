"""Derive the polynomial used for part of the softmax exponentials.

Method: Cody-Waite style range reduction x = j + f with j = round(x) and
f in [-1/2, 1/2], so 2^x = 2^j * 2^f; 2^j is applied by adding j to the
fp32 exponent field.  2^f is replaced by the degree-3 polynomial that
minimises the maximum RELATIVE error on [-1/2, 1/2], found with the Remez
exchange algorithm (equioscillation at n + 2 = 5 reference points).  The
coefficients are then rounded to fp32 and the fp32-evaluated error is
reported.  bf16 P (8 significant bits, relative spacing 2^-8) needs far less
than this accuracy; the test suite compares the kernel's polynomial against
CUDA's exp2f on the GPU.

    python causal_dit_kv_b200/csrc/gen_exp2_poly.py
"""
import numpy as np

DEG = 3
LO, HI = -0.5, 0.5


def remez(deg=DEG, iters=30):
    n = deg + 2
    # Chebyshev extrema as the initial reference
    ref = 0.5 * (LO + HI) + 0.5 * (HI - LO) * np.cos(np.pi * np.arange(n)[::-1] / (n - 1))
    grid = np.linspace(LO, HI, 200001)
    coef = None
    for _ in range(iters):
        # sum_k c_k x_i^k - 2^x_i = (-1)^i E 2^x_i
        A = np.zeros((n, n))
        for i, x in enumerate(ref):
            A[i, :deg + 1] = x ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) * 2.0 ** x
        sol = np.linalg.solve(A, 2.0 ** ref)
        coef = sol[:deg + 1]
        err = (np.polyval(coef[::-1], grid) - 2.0 ** grid) / 2.0 ** grid
        # new reference: extrema of err between sign changes
        sign = np.sign(err)
        idx = [0]
        for k in range(1, len(grid)):
            if sign[k] != sign[idx[-1]]:
                idx.append(k)
            elif abs(err[k]) > abs(err[idx[-1]]):
                idx[-1] = k
        if len(idx) < n:
            break
        # keep the n consecutive extrema with the largest minimum magnitude
        best = max(range(len(idx) - n + 1), key=lambda s: min(abs(err[idx[s:s + n]])))
        ref = grid[idx[best:best + n]]
    return coef


def main():
    coef = remez()
    c32 = coef.astype(np.float32)
    x = np.linspace(LO, HI, 1_000_001).astype(np.float32)
    p = np.float32(c32[3])
    for k in (2, 1, 0):
        p = (p * x + c32[k]).astype(np.float32)
    rel = np.abs(p.astype(np.float64) / 2.0 ** x.astype(np.float64) - 1.0)
    for k, c in enumerate(c32):
        print(f"c{k} = {float(c):.9e}f  (0x{np.float32(c).view(np.uint32):08x})")
    print(f"max relative error (fp32 Horner on [-1/2, 1/2]): {rel.max():.3e}")


if __name__ == "__main__":
    main()
