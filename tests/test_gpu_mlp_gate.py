"""The pages' bottleneck-MLP gate on the GPU (fused decode, separate EC pass, tcgen05) against the
oracle, through the C ABI: gamma(t) = sigmoid(W2 relu(W1 t + b1) + b2), u = alpha gamma t."""
import numpy as np
import pytest
import torch

import oracle
from synthetic import make_layer
from gpu_helpers import check_close, host_f64, to_dev, to_dev_bf16

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import w4_gemm_error_channel_b200 as spear
else:
    spear = None


def _gate(r, H, seed):
    rng = np.random.default_rng(seed)
    W1 = (rng.standard_normal((H, r)) * 0.5).astype(np.float32)
    b1 = (rng.standard_normal(H) * 0.2).astype(np.float32)
    W2 = (rng.standard_normal((r, H)) * 0.5).astype(np.float32)
    b2 = (rng.standard_normal(r) * 0.5).astype(np.float32)
    return W1, b1, W2, b2


def _run(L, M, H, alpha, plan_fix=None, y_dtype=torch.bfloat16):
    W1, b1, W2, b2 = _gate(L.rank, H, 7 + H)
    packed, scale, zero = spear.spear_pack_w4(to_dev(L.W))
    ec = spear.EC(to_dev_bf16(L.A_bits), to_dev_bf16(L.B_bits), to_dev_bf16(L.wg_bits), L.b_g,
                  gate_w1=to_dev(W1), gate_b1=to_dev(b1), gate_w2=to_dev(W2), gate_b2=to_dev(b2), alpha=alpha)
    plan = spear.spear_gemm_plan(M, L.N, L.K, L.rank)
    if plan_fix:
        plan_fix(plan)
    ws = spear.alloc_workspace(plan.workspace_bytes + (M * L.rank * 2 + 256) + min(M, 256) * L.N * 4)
    y = spear.spear_w4ec_gemm(to_dev_bf16(L.x(M)), packed, scale, zero, ec, y_dtype=y_dtype, plan=plan,
                              workspace=ws)
    torch.cuda.synchronize()
    assert spear.spear_get_device_status(ws) == 0
    p, s, z = oracle.pack_w4(L.W)
    ref = oracle.w4ec_gemm_mlp(L.x(M), p, s, z, L.A_bits, L.B_bits, W1, b1, W2, b2, alpha)
    return host_f64(y), ref, plan, ws


@pytest.mark.parametrize("M,r,H", [(1, 16, 4), (4, 64, 16), (16, 64, 64), (33, 32, 8)])
def test_mlp_gate_decode(M, r, H):
    L = make_layer("mlpd", 50 + M + r, M, 512, 1024, r, outlier_frac=0.01, outlier_scale=20.0, ec_std=0.05)
    y, ref, plan, ws = _run(L, M, H, 1.5)
    assert plan.kernel_id == spear.SPEAR_KERNEL_SPLITK
    check_close(y, ref, True, f"MLP gate decode M={M} r={r} H={H}")
    assert int(ws[: (128 + 1024) * 1024].count_nonzero().item()) == 0


def test_mlp_gate_separate_pass():
    L = make_layer("mlps", 61, 16, 512, 1024, 64, outlier_frac=0.01, outlier_scale=20.0, ec_std=0.05)

    def fix(p):
        p.flags = spear.SPEAR_PLAN_SEPARATE_EC
    y, ref, plan, _ = _run(L, 16, 16, 0.8, plan_fix=fix)
    check_close(y, ref, True, "MLP gate separate EC pass")


@pytest.mark.parametrize("M,r,H,tile_m", [(128, 64, 16, 128), (300, 128, 64, 256), (200, 32, 8, 160)])
def test_mlp_gate_tc05(M, r, H, tile_m):
    L = make_layer("mlpt", 70 + M + r, M, 256, 512, r, outlier_frac=0.01, outlier_scale=20.0, ec_std=0.05)

    def fix(p):
        p.kernel_id, p.tile_n, p.split_k, p.tile_m, p.flags = spear.SPEAR_KERNEL_TC05, 128, 1, tile_m, 0
    y, ref, plan, _ = _run(L, M, H, 1.2, plan_fix=fix)
    check_close(y, ref, True, f"MLP gate tcgen05 M={M} r={r} H={H}")


@pytest.mark.parametrize("M,split,tile_m", [(128, 2, 128), (300, 4, 128), (300, 8, 256)])
def test_mlp_gate_tc05_k_split(M, split, tile_m):
    # With the MLP gate the EC tiles keep the whole K range (one CTA per 128 tokens, padded to whole
    # clusters) while the main tiles split theirs.
    L = make_layer("mlpk", 90 + M + split, M, 256, 1024, 64, outlier_frac=0.01, outlier_scale=20.0, ec_std=0.05)

    def fix(p):
        p.kernel_id, p.tile_n, p.split_k, p.tile_m, p.flags = spear.SPEAR_KERNEL_TC05, 128, split, tile_m, 0
    y, ref, plan, ws = _run(L, M, 16, 1.2, plan_fix=fix)
    check_close(y, ref, True, f"MLP gate tcgen05 K split {split} M={M}")
    assert int(ws[: (128 + 1024) * 1024].count_nonzero().item()) == 0, "EC flags not re-armed"


def test_mlp_gate_fp32_and_limits():
    # fp32 output meets the literal bound; gamma = 0 (b2 = -inf, W2 = 0) gives the plain layer.
    L = make_layer("mlpf", 81, 8, 256, 512, 32, ec_std=0.05)
    y, ref, _, _ = _run(L, 8, 8, 1.0, y_dtype=torch.float32)
    check_close(y, ref, False, "MLP gate fp32")
    packed, scale, zero = spear.spear_pack_w4(to_dev(L.W))
    x = to_dev_bf16(L.x(8))
    W1, b1, _, _ = _gate(32, 8, 3)
    ec = spear.EC(to_dev_bf16(L.A_bits), to_dev_bf16(L.B_bits), to_dev_bf16(L.wg_bits), 0.0,
                  gate_w1=to_dev(W1), gate_b1=to_dev(b1), gate_w2=torch.zeros((32, 8), device="cuda"),
                  gate_b2=torch.full((32,), float("-inf"), device="cuda"))
    y_off = spear.spear_w4ec_gemm(x, packed, scale, zero, ec, y_dtype=torch.float32)
    y_plain = spear.spear_w4ec_gemm(x, packed, scale, zero, None, y_dtype=torch.float32,
                                    plan=spear.spear_gemm_plan(8, L.N, L.K, 32))
    assert torch.equal(y_off, y_plain)
