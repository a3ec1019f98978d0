"""Coefficients of the polynomial 2^f used by exp2_poly in tc_attn.cuh.

Minimax fit of 2^f on f in [-1/2, 1/2] in relative error by the Remez
exchange algorithm (mpmath, 40 digits), then a check of the fp32 fused
multiply-add Horner evaluation against exact 2^f.  Run:
    python fit_exp2.py 5
and paste the printed coefficients (c0 .. c5) into tc_attn.cuh.
"""
import numpy as np, mpmath as mp
mp.mp.dps = 40
deg = int(__import__('sys').argv[1]) if len(__import__('sys').argv) > 1 else 6
a, b = -0.5, 0.5
f = lambda x: mp.power(2, x)
# Remez for relative error: minimize max |(p(x) - 2^x) / 2^x|
n = deg
xs = [ (a+b)/2 + (b-a)/2 * mp.cos(mp.pi * (n + 1 - i) / (n + 1)) for i in range(n + 2)]
for it in range(30):
    # solve p(x_i) - f(x_i) = (-1)^i E f(x_i)
    A = mp.matrix(n + 2, n + 2); rhs = mp.matrix(n + 2, 1)
    for i, x in enumerate(xs):
        for j in range(n + 1): A[i, j] = x ** j
        A[i, n + 1] = -((-1) ** i) * f(x)
        rhs[i] = f(x)
    sol = mp.lu_solve(A, rhs)
    c = [sol[j] for j in range(n + 1)]; E = sol[n + 1]
    err = lambda x: (sum(c[j] * x ** j for j in range(n + 1)) - f(x)) / f(x)
    grid = [a + (b - a) * k / 4000 for k in range(4001)]
    vals = [err(x) for x in grid]
    # new extrema: pick sign-alternating local extrema
    ext = []
    for k in range(len(grid)):
        v = vals[k]
        l = vals[k - 1] if k > 0 else -v
        r = vals[k + 1] if k < len(grid) - 1 else -v
        if (abs(v) >= abs(l) and abs(v) >= abs(r)):
            ext.append((grid[k], v))
    # keep n+2 alternating extrema with largest magnitude
    alt = []
    for x, v in ext:
        if alt and mp.sign(alt[-1][1]) == mp.sign(v):
            if abs(v) > abs(alt[-1][1]): alt[-1] = (x, v)
        else:
            alt.append((x, v))
    while len(alt) > n + 2:
        if abs(alt[0][1]) < abs(alt[-1][1]): alt.pop(0)
        else: alt.pop()
    if len(alt) == n + 2: xs = [x for x, _ in alt]
maxerr = max(abs(v) for v in vals)
print("deg", deg, "max rel approx error", float(maxerr))
cf = [np.float32(float(x)) for x in c]
print("coeffs:", ["%.9e" % float(x) for x in cf])
# fp32 Horner simulation over a dense grid
fs = np.linspace(-0.5, 0.5, 2000001, dtype=np.float32)
acc = np.full_like(fs, cf[-1])
for j in range(deg - 1, -1, -1):
    acc = (acc * fs + cf[j]).astype(np.float32)   # fma not exact in numpy, close enough (checks below with float64 fma)
exact = np.exp2(fs.astype(np.float64))
rel = np.abs(acc.astype(np.float64) - exact) / exact
print("fp32 Horner max rel err", rel.max(), "ulps(2^-23)", rel.max() / 2 ** -23)
# with true fma (evaluate in float64 then round each step to fp32)
acc2 = np.full(fs.shape, np.float64(cf[-1]))
for j in range(deg - 1, -1, -1):
    acc2 = np.float32(acc2 * fs.astype(np.float64) + np.float64(cf[j])).astype(np.float64)
rel2 = np.abs(acc2 - exact) / exact
print("fp32 FMA Horner max rel err", rel2.max(), "ulps", rel2.max() / 2 ** -23)
