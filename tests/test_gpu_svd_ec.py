"""Static SVD-initialised compensator: the library's initialiser and the layer with its factors.

* The initialiser's factors (cuSOLVER on the device) against the oracle's fp64 SVD: the products
  A B agree within the bf16 rounding of the factors (singular vectors are unique only up to sign,
  the product is unique when the singular values are distinct).
* The layer with the oracle's factors (bf16, gate held at 1) against the oracle, through the C ABI.
* The share of the 4-bit output error it removes, measured on the GPU output, matches the
  oracle's, is positive and grows with the rank.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import svd_ec
from synthetic import bf16_bits_from_f32, f32_from_bf16_bits, make_layer
from gpu_helpers import check_close, host_f64, to_dev, to_dev_bf16

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import w4_gemm_error_channel_b200 as spear
    from w4_gemm_error_channel_b200.svd_init import svd_compensator
else:
    spear = None


def _layer():
    return make_layer("svdg", 23, 16, 512, 1024, 0, outlier_frac=0.01, outlier_scale=20.0)


@pytest.mark.parametrize("r", [16, 64])
def test_initialiser_matches_oracle_svd(r):
    L = _layer()
    W = to_dev(L.W)
    packed, scale, zero = spear.spear_pack_w4(W)
    ec = svd_compensator(W, packed, scale, zero, r)
    AB = (ec.A.double() @ ec.B.double()).cpu().numpy()
    p, s, z = oracle.pack_w4(L.W)
    A, B, sv = svd_ec.svd_factors(svd_ec.weight_error_t(L.W, p, s, z), r)
    ref = A @ B
    assert sv[r - 1] > sv[r] * (1 + 1e-6)                  # the rank-r subspace is unique
    err = np.linalg.norm(AB - ref) / np.linalg.norm(ref)
    assert err < 1e-2, err
    assert ec.b_g == float("inf") and int(torch.count_nonzero(ec.w_g)) == 0


def test_layer_with_svd_factors_and_gap():
    L = _layer()
    W = to_dev(L.W)
    packed, scale, zero = spear.spear_pack_w4(W)
    p, s, z = oracle.pack_w4(L.W)
    E_t = svd_ec.weight_error_t(L.W, p, s, z)
    M = L.x_bits.shape[0]
    x = to_dev_bf16(L.x(M))
    xf = f32_from_bf16_bits(L.x(M)).astype(np.float64)
    y_fp = xf @ L.W.astype(np.float64).T
    y_w4 = oracle.w4ec_gemm(L.x(M), p, s, z)
    wg_bits = np.zeros(L.K, dtype=np.uint16)
    gaps = []
    for r in (16, 64, 256):
        A, B, _ = svd_ec.svd_factors(E_t, r)
        A_bits, B_bits = bf16_bits_from_f32(A), bf16_bits_from_f32(B)
        ref = oracle.w4ec_gemm(L.x(M), p, s, z, A_bits, B_bits, wg_bits, float("inf"))
        ec = spear.EC(to_dev_bf16(A_bits), to_dev_bf16(B_bits), to_dev_bf16(wg_bits), float("inf"))
        y = host_f64(spear.spear_w4ec_gemm(x, packed, scale, zero, ec, y_dtype=torch.float32))
        check_close(y, ref, False, f"svd EC r={r}")
        g_gpu, g_ref = svd_ec.gap_recovered(y, y_fp, y_w4), svd_ec.gap_recovered(ref, y_fp, y_w4)
        assert abs(g_gpu - g_ref) < 1e-3, (r, g_gpu, g_ref)
        gaps.append(g_gpu)
    assert 0.0 < gaps[0] < gaps[1] < gaps[2], gaps
