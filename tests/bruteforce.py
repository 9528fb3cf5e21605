"""FP64 brute force of the gated delta rule, in matrix form (test helper).

This is the transition the pages write for the two layer kinds, evaluated
with float64 matrix products and no quantization:

    GDN:  S <- alpha (I - beta k k^T) S + beta k v^T
    KDA:  S <- (I - beta k k^T) Diag(alpha) S + beta k v^T
    readout o = S^T q   (STEPQuant Appendix Table C2, step 3)

It is deliberately the product form, not the expanded per-element form the
oracle uses (STEPQuant Table C2, step 2), so that agreement between the two
checks the algebra rather than restating it.
"""
import numpy as np


def step(S, q, k, v, alpha, beta):
    S = np.asarray(S, np.float64)
    dk = S.shape[0]
    k = np.asarray(k, np.float64).reshape(dk, 1)
    q = np.asarray(q, np.float64).reshape(dk)
    v = np.asarray(v, np.float64).reshape(1, -1)
    a = np.asarray(alpha, np.float64).reshape(-1)
    D = np.diag(a if a.size == dk else np.full(dk, a[0]))
    P = np.eye(dk) - float(beta) * (k @ k.T)
    Sn = P @ D @ S + float(beta) * (k @ v)
    return Sn, Sn.T @ q


def round_f16(x):
    """Round float64 to binary16 (numpy's conversion, nearest even)."""
    return np.asarray(x, np.float64).astype(np.float16)
