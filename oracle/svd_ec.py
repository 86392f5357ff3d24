"""Static SVD-initialised error compensator in fp64.

TEST INFRASTRUCTURE, like the rest of ``oracle/``: only the tests use it, and the CUDA library
never does.

SPEAR technical summary, section 1: the post-quantisation compensators that precede SPEAR apply
one static low-rank correction to every token; section 3.1 reports how much of the gap between
the 4-bit and the full-precision model a compensator recovers.  The data-free static compensator
of rank r is the best rank-r approximation, in the Frobenius norm (Eckart-Young), of the weight
error seen from the layer's input side:

    (W - W_hat)^T  ~=  A B,    A = U_r diag(sqrt(s_r)),  B = diag(sqrt(s_r)) V_r^T,

from the singular value decomposition (W - W_hat)^T = U diag(s) V^T, with the gate held at 1
(w_g = 0, b_g = +inf), so that y = x W_hat^T + x A B.  The SVD is numpy's (LAPACK), a library
primitive used as one step.
"""
from __future__ import annotations

import numpy as np

from . import default as _default


def weight_error_t(W: np.ndarray, packed: np.ndarray, s_bits: np.ndarray, z_bits: np.ndarray) -> np.ndarray:
    """(W - W_hat)^T in fp64, [K, N]; W_hat from the oracle's exact dequantisation."""
    K = W.shape[1]
    W_hat = _default().dequant_w4(packed, s_bits, z_bits, K)
    return (np.asarray(W, dtype=np.float64) - W_hat).T


def svd_factors(E_t: np.ndarray, rank: int):
    """A [K, r], B [r, N] (fp64) and every singular value of E_t, largest first."""
    U, s, Vt = np.linalg.svd(E_t, full_matrices=False)
    root = np.sqrt(s[:rank])
    return U[:, :rank] * root, root[:, None] * Vt[:rank], s


def gap_recovered(y: np.ndarray, y_fp: np.ndarray, y_w4: np.ndarray) -> float:
    """Share of the 4-bit layer's output error removed: 1 - |y - y_fp|_F / |y_w4 - y_fp|_F."""
    return 1.0 - float(np.linalg.norm(y - y_fp) / np.linalg.norm(y_w4 - y_fp))
