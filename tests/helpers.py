"""Error metrics shared by the parity tests.

max_rel   = max|x - r| / max|r| over a whole tensor (outputs);
frob_rel  = ||x - r||_F / ||r||_F (states).
"""
import numpy as np


def max_rel(x, r):
    x = np.asarray(x, dtype=np.float64)
    r = np.asarray(r, dtype=np.float64)
    den = np.max(np.abs(r))
    num = np.max(np.abs(x - r))
    return float(num / den) if den > 0 else float(num)


def frob_rel(x, r):
    x = np.asarray(x, dtype=np.float64)
    r = np.asarray(r, dtype=np.float64)
    den = np.linalg.norm(r.ravel())
    num = np.linalg.norm((x - r).ravel())
    return float(num / den) if den > 0 else float(num)
