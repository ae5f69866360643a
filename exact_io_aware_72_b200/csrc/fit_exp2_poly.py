"""Fit the polynomial the forward kernel uses for part of its 2^x evaluations.

Method: Cody-Waite style range reduction x = n + f with n = round(x) and
f in [-1/2, 1/2], then 2^x = 2^n * q(f) where q is the degree-3 polynomial
minimising the maximum RELATIVE error of q(f) against 2^f on [-1/2, 1/2],
found with the Remez exchange algorithm.  Run it to reprint the coefficients
and their error; the kernel's table (attn_fwd_kernel.cuh, kExp2Poly*) holds the
degree-3 line rounded to float32.
"""
import numpy as np
def remez(n, a=-0.5, b=0.5, iters=40):
    m = n + 2
    x = np.cos(np.pi * np.arange(m)[::-1] / (m - 1)) * (b - a) / 2 + (a + b) / 2
    f = lambda t: np.exp2(t)
    for _ in range(iters):
        # solve sum c_k x^k - f(x) = (-1)^i E f(x)  (relative error)
        A = np.zeros((m, m))
        for i in range(m):
            A[i, :n + 1] = x[i] ** np.arange(n + 1)
            A[i, n + 1] = (-1) ** i * f(x[i])
        sol = np.linalg.solve(A, f(x))
        c, E = sol[:n + 1], sol[n + 1]
        t = np.linspace(a, b, 200001)
        err = (np.polyval(c[::-1], t) - f(t)) / f(t)
        # new extrema: sign-alternating maxima between zero crossings
        s = np.sign(err)
        idx = np.where(np.diff(s) != 0)[0]
        bounds = np.concatenate([[0], idx + 1, [len(t)]])
        ext = [seg_start + np.argmax(np.abs(err[seg_start:seg_end])) for seg_start, seg_end in zip(bounds[:-1], bounds[1:])]
        if len(ext) != m:
            break
        x = t[ext]
    return c, np.max(np.abs(err))
if __name__ == "__main__":
    for n in (2, 3, 4):
        c, e = remez(n)
        print(n, [float(np.float32(v)) for v in c], f"max rel err {e:.3e} (~2^{np.log2(e):.1f})")
