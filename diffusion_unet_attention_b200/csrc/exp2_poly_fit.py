import numpy as np
from scipy.optimize import linprog
f = np.linspace(-0.5, 0.5, 4001)
y = np.exp2(f)
for deg in (3, 4):
    n = deg + 1
    V = np.vander(f, n, increasing=True)          # c0 + c1 f + ...
    # minimize t s.t. -t*y <= V c - y <= t*y
    A1 = np.hstack([V, -y[:, None]]); b1 = y
    A2 = np.hstack([-V, -y[:, None]]); b2 = -y
    res = linprog(np.r_[np.zeros(n), 1.0], A_ub=np.vstack([A1, A2]), b_ub=np.r_[b1, b2],
                  bounds=[(None, None)] * n + [(0, None)], method="highs")
    c = res.x[:n]
    c32 = c.astype(np.float32)
    # evaluate in fp32 Horner like the kernel
    ff = np.linspace(-0.5, 0.5, 200001).astype(np.float32)
    p = np.full_like(ff, c32[-1])
    for k in range(n - 2, -1, -1):
        p = (p * ff + c32[k]).astype(np.float32)
    rel = np.abs(p.astype(np.float64) / np.exp2(ff.astype(np.float64)) - 1).max()
    print(deg, [float(x) for x in c32], "lp max rel", res.x[-1], "fp32 horner max rel", rel)
