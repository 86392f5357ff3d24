"""Group-wise scales on the GPU against the oracle, through the C ABI: the packer bit for bit, and
the layer (grouped weight-streaming kernel; with a compensator, the EC tiles beside it and the
up-projection join) within the layer tolerance."""
import numpy as np
import pytest
import torch

import oracle
from synthetic import bf16_bits_from_f32, f32_from_bf16_bits, make_layer
from gpu_helpers import check_close, f16_bits, host_f64, to_dev, to_dev_bf16

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import w4_gemm_error_channel_b200 as spear
else:
    spear = None

ZEROED = (128 + 1024) * 1024


@pytest.mark.parametrize("G", [128, 256, 64])
@pytest.mark.parametrize("bf16_in", [False, True])
def test_grouped_pack_bit_exact(G, bf16_in):
    L = make_layer("gpack", 200 + G, 1, 256, 1024, 0, outlier_frac=0.02, outlier_scale=10.0)
    W = L.W
    if bf16_in:
        W = f32_from_bf16_bits(bf16_bits_from_f32(W))
        Wd = to_dev_bf16(bf16_bits_from_f32(L.W))
    else:
        Wd = to_dev(W)
    packed, scale, zero = spear.spear_pack_w4_grouped(Wd, G)
    p, s, z = oracle.pack_w4_grouped(W, G)
    assert np.array_equal(packed.cpu().numpy(), p)
    assert np.array_equal(f16_bits(scale), s) and np.array_equal(f16_bits(zero), z)


def _run(L, M, G, ec_on=True, y_dtype=torch.bfloat16, b_g=None, mlp=None):
    packed, scale, zero = spear.spear_pack_w4_grouped(to_dev(L.W), G)
    bg = L.b_g if b_g is None else b_g
    ec = None
    if ec_on:
        kw = {}
        if mlp is not None:
            W1, b1, W2, b2, alpha = mlp
            kw = dict(gate_w1=to_dev(W1), gate_b1=to_dev(b1), gate_w2=to_dev(W2), gate_b2=to_dev(b2), alpha=alpha)
        ec = spear.EC(to_dev_bf16(L.A_bits), to_dev_bf16(L.B_bits), to_dev_bf16(L.wg_bits), bg, **kw)
    ws = spear.alloc_workspace(spear.spear_grouped_workspace_bytes(M, L.N, L.K, G, L.rank if ec_on else 0))
    y = spear.spear_w4ec_gemm_grouped(to_dev_bf16(L.x(M)), packed, scale, zero, G, ec, y_dtype=y_dtype, workspace=ws)
    torch.cuda.synchronize()
    assert spear.spear_get_device_status(ws) == 0
    assert int(ws[:ZEROED].count_nonzero().item()) == 0
    return host_f64(y)


def _ref(L, M, G, ec_on=True, b_g=None, rows=None):
    p, s, z = oracle.pack_w4_grouped(L.W, G)
    xs = L.x(M) if rows is None else L.x(M)[rows]
    if not ec_on:
        return oracle.w4ec_gemm_grouped(xs, p, s, z, G)
    return oracle.w4ec_gemm_grouped(xs, p, s, z, G, L.A_bits, L.B_bits, L.wg_bits, L.b_g if b_g is None else b_g)


@pytest.mark.parametrize("G", [128, 512])
@pytest.mark.parametrize("r", [0, 16, 64, 128])
@pytest.mark.parametrize("M", [1, 5, 16, 33, 300])
def test_grouped_layer(M, r, G):
    L = make_layer("grp", 300 + M + r + G, M, 384, 1024, max(r, 16), outlier_frac=0.01, outlier_scale=20.0, b_g=0.2)
    y = _run(L, M, G, ec_on=r > 0)
    check_close(y, _ref(L, M, G, ec_on=r > 0), True, f"grouped M={M} r={r} G={G}")


def test_grouped_fp32_gate_off_and_per_channel_limit():
    L = make_layer("grpf", 41, 64, 256, 512, 32, b_g=-0.5)
    check_close(_run(L, 64, 128, y_dtype=torch.float32), _ref(L, 64, 128), False, "grouped fp32")
    # b_g = -inf: g = 0, so the layer equals the plain grouped layer from the same kernel.
    off = _run(L, 64, 128, b_g=float("-inf"))
    plain = _run(L, 64, 128, ec_on=False)
    assert np.array_equal(off, plain)
    # G = K: the per-channel layer (same codes and scales as spear_pack_w4).
    packed, scale, zero = spear.spear_pack_w4_grouped(to_dev(L.W), 512)
    p1, s1, z1 = spear.spear_pack_w4(to_dev(L.W))
    assert torch.equal(packed, p1) and torch.equal(scale[:, 0], s1) and torch.equal(zero[:, 0], z1)
    check_close(_run(L, 64, 512, ec_on=False), oracle.w4ec_gemm(L.x(64), *oracle.pack_w4(L.W)), True, "G = K")


def test_grouped_mlp_gate():
    L = make_layer("grpm", 51, 40, 256, 512, 32, ec_std=0.05)
    rng = np.random.default_rng(52)
    H = 8
    W1 = (rng.standard_normal((H, 32)) * 0.5).astype(np.float32)
    b1 = (rng.standard_normal(H) * 0.2).astype(np.float32)
    W2 = (rng.standard_normal((32, H)) * 0.5).astype(np.float32)
    b2 = (rng.standard_normal(32) * 0.5).astype(np.float32)
    y = _run(L, 40, 128, mlp=(W1, b1, W2, b2, 1.1))
    # The oracle: grouped main term + the MLP-gated compensator (its plain-layer part cancels).
    p, s, z = oracle.pack_w4_grouped(L.W, 128)
    main = oracle.w4ec_gemm_grouped(L.x(40), p, s, z, 128)
    pc, sc, zc = oracle.pack_w4(L.W)
    ec = (oracle.w4ec_gemm_mlp(L.x(40), pc, sc, zc, L.A_bits, L.B_bits, W1, b1, W2, b2, 1.1)
          - oracle.w4ec_gemm(L.x(40), pc, sc, zc))
    check_close(y, main + ec, True, "grouped MLP gate")


@pytest.mark.parametrize("M", [16, 2048])
def test_grouped_decode_qo_shape_sampled(M):
    L = make_layer("grpq", 61, M, 4096, 4096, 64, outlier_frac=0.01, outlier_scale=20.0)
    rows = np.array([0, 1, M // 2, M - 1])
    y = _run(L, M, 128)
    check_close(y[rows], _ref(L, M, 128, rows=rows), True, f"grouped 4096x4096 M={M}")
