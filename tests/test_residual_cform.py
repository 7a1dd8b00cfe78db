"""The walk on the GPU keeps the renormalised residual in closed form: after
the j-th rejected sibling at a node the distribution is max(0, p - c_j q) / Z_j
with c_1 = 1, c_{j+1} = c_j + Z_j and Z_j = sum max(0, p - c_j q), instead of
renormalising a stored row each time (blog "Speculative decoding x tree
attention", section 2: on rejection resample from max(0, p - q) normalised).
This checks the algebra in fp64 against the literal repeated renormalisation,
and that the acceptance test r < P_j(x) / q(x) is the same decision as
r * Z_j * q(x) < max(0, p(x) - c_j q(x))."""
import numpy as np


def test_closed_form_residual_equals_repeated_renormalisation():
    rng = np.random.default_rng(11)
    for _ in range(200):
        V = int(rng.integers(2, 400))
        p = rng.dirichlet(np.ones(V) * rng.uniform(0.05, 2.0))
        q = rng.dirichlet(np.ones(V) * rng.uniform(0.05, 2.0))
        P = p.copy()
        c = 0.0
        for _ in range(int(rng.integers(1, 8))):
            # literal: one more rejection renormalises max(0, P - q)
            R = np.maximum(0.0, P - q)
            if R.sum() <= 0.0:
                break
            P = R / R.sum()
            # closed form: c advances by the previous mass, starting from 1
            c = 1.0 if c == 0.0 else c + Z
            r = np.maximum(0.0, p - c * q)
            Z = r.sum()
            np.testing.assert_allclose(r / Z, P, rtol=1e-9, atol=1e-12)
            # the acceptance decision for any candidate token and uniform
            x = int(rng.integers(0, V))
            u = rng.random()
            if q[x] > 0 and abs(u - P[x] / q[x]) > 1e-9:
                assert (u < P[x] / q[x]) == (u * Z * q[x] < r[x])
