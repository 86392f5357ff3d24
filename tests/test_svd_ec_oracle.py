"""Pins for the static SVD-initialised compensator of the oracle (oracle/svd_ec.py), on the CPU.

Each check compares the oracle with something computed independently of it:
* full rank: A B reproduces (W - W_hat)^T, which is built here from the oracle's unpacked codes,
  scales and zero-points by plain numpy arithmetic;
* Eckart-Young: the rank-r residual equals the energy of the discarded singular values, where
  those come from a separate LAPACK call on W - W_hat (not its transpose);
* the top singular value agrees with power iteration on E^T E;
* the compensated layer from the C oracle (gate held at 1 by w_g = 0, b_g = +inf) equals
  x W_hat^T + x A B from numpy matmuls;
* gap recovered is 1 at full rank (fp64 factors), 0 at rank 0, and never decreases with rank.
"""
import numpy as np

import oracle
from oracle import svd_ec
from synthetic import bf16_bits_from_f32, f32_from_bf16_bits, make_layer


def _layer():
    return make_layer("svd", 17, 6, 48, 64, 0, outlier_frac=0.05, outlier_scale=10.0)


def _error_t(L):
    packed, s_bits, z_bits = oracle.pack_w4(L.W)
    q = oracle.unpack_nibbles(packed, L.K).astype(np.float64)
    s = np.array([oracle.f16_bits_to_f64(int(b)) for b in s_bits])
    z = np.array([oracle.f16_bits_to_f64(int(b)) for b in z_bits])
    W_hat = (q - z[:, None]) * s[:, None]
    return packed, s_bits, z_bits, (L.W.astype(np.float64) - W_hat).T


def test_error_matrix_matches_numpy_dequant():
    L = _layer()
    packed, s_bits, z_bits, E_ref = _error_t(L)
    assert np.array_equal(svd_ec.weight_error_t(L.W, packed, s_bits, z_bits), E_ref)


def test_full_rank_reproduces_the_error():
    L = _layer()
    _, _, _, E_t = _error_t(L)
    A, B, _ = svd_ec.svd_factors(E_t, min(E_t.shape))
    assert np.allclose(A @ B, E_t, rtol=0, atol=1e-12 * np.abs(E_t).max())


def test_eckart_young_residual_and_top_value():
    L = _layer()
    _, _, _, E_t = _error_t(L)
    s_other = np.linalg.svd(E_t.T, compute_uv=False)           # separate call, other shape
    v = np.ones(E_t.shape[1])
    for _ in range(2000):                                        # power iteration on E^T E
        v = E_t.T @ (E_t @ v)
        v /= np.linalg.norm(v)
    top = np.linalg.norm(E_t @ v)
    for r in (1, 5, 17):
        A, B, s = svd_ec.svd_factors(E_t, r)
        res = np.linalg.norm(E_t - A @ B) ** 2
        assert abs(res - np.sum(s_other[r:] ** 2)) <= 1e-10 * np.sum(s_other ** 2)
    assert abs(s[0] - top) <= 1e-9 * top


def test_compensated_layer_and_gap():
    L = _layer()
    packed, s_bits, z_bits, E_t = _error_t(L)
    x = f32_from_bf16_bits(L.x_bits).astype(np.float64)
    W_hat = L.W.astype(np.float64) - E_t.T
    y_fp = x @ L.W.astype(np.float64).T
    y_w4 = x @ W_hat.T
    gaps = []
    for r in (0, 4, 16, 48):
        A, B, _ = svd_ec.svd_factors(E_t, r)
        if r == 0:
            y = y_w4
        else:
            A_bits, B_bits = bf16_bits_from_f32(A), bf16_bits_from_f32(B)
            wg_bits = np.zeros(L.K, dtype=np.uint16)
            y = oracle.w4ec_gemm(L.x_bits, packed, s_bits, z_bits, A_bits, B_bits, wg_bits, float("inf"))
            ref = y_w4 + x @ (f32_from_bf16_bits(A_bits).astype(np.float64) @ f32_from_bf16_bits(B_bits))
            assert np.allclose(y, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())
        gaps.append(svd_ec.gap_recovered(y, y_fp, y_w4))
    assert gaps[0] == 0.0
    assert all(b >= a - 1e-12 for a, b in zip(gaps, gaps[1:])), gaps
    A, B, _ = svd_ec.svd_factors(E_t, min(E_t.shape))
    assert abs(svd_ec.gap_recovered(y_w4 + x @ (A @ B), y_fp, y_w4) - 1.0) < 1e-9
