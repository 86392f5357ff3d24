"""The tcgen05 (TMEM) prefill kernel against the CPU oracle, through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
from synthetic import config_layers, make_layer
from gpu_helpers import check_close, host_f64, to_dev, to_dev_bf16

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import w4_gemm_error_channel_b200 as spear
else:
    spear = None


def tc_plan(M, N, K, tile_m, wrows=128, split=1):
    p = spear.spear_gemm_plan(M, N, K, 0)
    p.kernel_id = spear.SPEAR_KERNEL_TC05
    p.tile_n, p.split_k, p.tile_m = wrows, split, tile_m
    return p


def run(L, M, tile_m, y_dtype=torch.bfloat16, rows=None, wrows=128, split=1):
    W = to_dev(L.W)
    packed, scale, zero = spear.spear_pack_w4(W)
    x = to_dev_bf16(L.x(M))
    ws = spear.alloc_workspace(spear.spear_gemm_plan(M, L.N, L.K, 0).workspace_bytes)
    y = spear.spear_w4ec_gemm(x, packed, scale, zero, None, y_dtype=y_dtype,
                              plan=tc_plan(M, L.N, L.K, tile_m, wrows, split), workspace=ws)
    torch.cuda.synchronize()
    assert spear.spear_get_device_status(ws) == 0
    p, s, z = oracle.pack_w4(L.W)
    xs = L.x(M) if rows is None else L.x(M)[rows]
    ref = oracle.w4ec_gemm(xs, p, s, z)
    got = host_f64(y) if rows is None else host_f64(y)[rows]
    return got, ref


@pytest.mark.parametrize("tile_m", [128, 160, 192, 256])
@pytest.mark.parametrize("M", [1, 77, 128, 129, 300, 512])
def test_tc05_small(M, tile_m):
    L = make_layer("tc", 5 + M, M, 384, 448, 0, outlier_frac=0.02, outlier_scale=10.0)
    got, ref = run(L, M, tile_m)
    check_close(got, ref, True, f"tc05 M={M} tile_m={tile_m}")


def test_tc05_fp32_output():
    L = make_layer("tc", 9, 200, 256, 1024, 0)
    got, ref = run(L, 200, 128, y_dtype=torch.float32)
    check_close(got, ref, False, "tc05 fp32")


@pytest.mark.parametrize("tile_m", [128, 160, 192, 256])
def test_tc05_prefill_shape_sampled(tile_m):
    L = config_layers(3)[0]
    rows = np.array([0, 1, 255, 256, 1031, 2047])
    got, ref = run(L, 2048, tile_m, rows=rows)
    check_close(got, ref, True, f"tc05 prefill tile_m={tile_m}")


@pytest.mark.parametrize("li", [0, 1, 2, 3])
def test_tc05_sweep_layer_without_ec(li):
    L = config_layers(4, M=4096, layers=(2,))[li]     # layer 2 carries no compensator
    rows = np.array([0, 100, 2049, 4095])
    got, ref = run(L, 4096, 256, rows=rows)
    check_close(got, ref, True, f"tc05 sweep L2.{li}")


def run_ec(L, M, tile_m, rows=None, b_g=None, y_dtype=torch.bfloat16, wrows=128, split=1):
    W = to_dev(L.W)
    packed, scale, zero = spear.spear_pack_w4(W)
    x = to_dev_bf16(L.x(M))
    bg = L.b_g if b_g is None else b_g
    ec = spear.EC(to_dev_bf16(L.A_bits), to_dev_bf16(L.B_bits), to_dev_bf16(L.wg_bits), bg)
    plan = spear.spear_gemm_plan(M, L.N, L.K, L.rank)
    plan.kernel_id, plan.tile_n, plan.split_k, plan.tile_m = spear.SPEAR_KERNEL_TC05, wrows, split, tile_m
    ws = spear.alloc_workspace(plan.workspace_bytes + (M * L.rank * 2 + 256))
    y = spear.spear_w4ec_gemm(x, packed, scale, zero, ec, y_dtype=y_dtype, plan=plan, workspace=ws)
    torch.cuda.synchronize()
    assert spear.spear_get_device_status(ws) == 0
    p, s, z = oracle.pack_w4(L.W)
    xs = L.x(M) if rows is None else L.x(M)[rows]
    ref = oracle.w4ec_gemm(xs, p, s, z, L.A_bits, L.B_bits, L.wg_bits, bg)
    got = host_f64(y) if rows is None else host_f64(y)[rows]
    return got, ref, y, ws


@pytest.mark.parametrize("tile_m", [128, 160, 192, 256])
@pytest.mark.parametrize("r", [16, 32, 48, 64, 128])
@pytest.mark.parametrize("M", [128, 300])
def test_tc05_ec_small(M, r, tile_m):
    L = make_layer("tcec", 11 + r + M, M, 256, 512, r, outlier_frac=0.02, outlier_scale=10.0, b_g=0.3)
    got, ref, _, ws = run_ec(L, M, tile_m)
    check_close(got, ref, True, f"tc05 EC M={M} r={r} tile_m={tile_m}")
    # Token tiles of 160 or 192 share 128-token EC blocks; every flag must still be re-armed.
    assert int(ws[: (128 + 1024) * 1024].count_nonzero().item()) == 0, "EC flags not re-armed"


def test_tc05_ec_fp32_and_gate_off():
    L = make_layer("tcec", 21, 200, 384, 640, 64, b_g=-1.0)
    got, ref, _, _ = run_ec(L, 200, 128, y_dtype=torch.float32)
    check_close(got, ref, False, "tc05 EC fp32")
    # b_g = -inf: g = 0 exactly, so the compensated layer equals the plain one bit for bit.
    _, _, y_off, _ = run_ec(L, 200, 128, b_g=float("-inf"))
    plain, _ = run(L, 200, 128)
    assert np.array_equal(host_f64(y_off), plain)


@pytest.mark.parametrize("tile_m", [128, 160, 192, 256])
def test_tc05_ec_prefill_sampled(tile_m):
    L = config_layers(3)[0]
    rows = np.array([0, 1, 255, 256, 1031, 2047])
    got, ref, _, ws = run_ec(L, 2048, tile_m, rows=rows)
    check_close(got, ref, True, f"tc05 EC prefill tile_m={tile_m}")
    zeroed = ws[: (128 + 1024) * 1024].cpu()
    assert int(zeroed.count_nonzero()) == 0, "EC flags not re-armed"


@pytest.mark.parametrize("li", [0, 3])
def test_tc05_ec_sweep_layer(li):
    L = config_layers(4, M=4096, layers=(0,))[li]     # layer 0 carries a rank-32 compensator
    rows = np.array([0, 100, 2049, 4095])
    got, ref, _, _ = run_ec(L, 4096, 256, rows=rows)
    check_close(got, ref, True, f"tc05 EC sweep L0.{li}")


# 256 weight rows per tile: two 128-row sub-tiles share every x stage.
@pytest.mark.parametrize("M", [1, 77, 300])
def test_tc05_256rows_small(M):
    L = make_layer("tc2", 31 + M, M, 768, 448, 0, outlier_frac=0.02, outlier_scale=10.0)
    got, ref = run(L, M, 128, wrows=256)
    check_close(got, ref, True, f"tc05 256 rows M={M}")


@pytest.mark.parametrize("r", [16, 64, 128])
@pytest.mark.parametrize("M", [128, 300])
def test_tc05_256rows_ec_small(M, r):
    L = make_layer("tc2ec", 41 + r + M, M, 512, 512, r, outlier_frac=0.02, outlier_scale=10.0, b_g=0.3)
    got, ref, _, ws = run_ec(L, M, 128, wrows=256)
    check_close(got, ref, True, f"tc05 256 rows EC M={M} r={r}")
    assert int(ws[: (128 + 1024) * 1024].count_nonzero().item()) == 0, "EC flags not re-armed"


def test_tc05_256rows_prefill_sampled():
    L = config_layers(3)[0]
    rows = np.array([0, 1, 255, 256, 1031, 2047])
    got, ref = run(L, 2048, 128, rows=rows, wrows=256)
    check_close(got, ref, True, "tc05 256 rows prefill")
    got, ref, _, _ = run_ec(L, 2048, 128, rows=rows, wrows=256)
    check_close(got, ref, True, "tc05 256 rows EC prefill")


# K split over a cluster of 2, 4 or 8 CTAs per tile; the partial tiles meet in shared memory.
@pytest.mark.parametrize("split", [2, 4, 8])
@pytest.mark.parametrize("tile_m", [128, 256])
@pytest.mark.parametrize("M", [1, 77, 300])
def test_tc05_k_split_small(M, tile_m, split):
    L = make_layer("tcks", 51 + M + split, M, 384, 1024, 0, outlier_frac=0.02, outlier_scale=10.0)
    got, ref = run(L, M, tile_m, split=split)
    check_close(got, ref, True, f"tc05 K split {split} M={M} tile_m={tile_m}")


@pytest.mark.parametrize("split", [2, 4, 8])
@pytest.mark.parametrize("r", [16, 64, 128])
@pytest.mark.parametrize("M", [128, 300])
def test_tc05_k_split_ec_small(M, r, split):
    L = make_layer("tcksec", 61 + r + M + split, M, 256, 1024, r, outlier_frac=0.02, outlier_scale=10.0, b_g=0.3)
    got, ref, _, ws = run_ec(L, M, 128, split=split)
    check_close(got, ref, True, f"tc05 K split {split} EC M={M} r={r}")
    assert int(ws[: (128 + 1024) * 1024].count_nonzero().item()) == 0, "EC flags not re-armed"


def test_tc05_k_split_odd_tiles_fp32_and_determinism():
    # 160- and 192-token tiles (owners of 80 and 48 tokens), fp32 output, and the fixed summation
    # order: two runs give the same bits.
    L = make_layer("tcks2", 71, 330, 384, 768, 32, b_g=0.1)
    for tile_m, split in ((160, 2), (192, 4), (192, 2)):
        got, ref, y1, _ = run_ec(L, 330, tile_m, split=split, y_dtype=torch.float32)
        check_close(got, ref, False, f"tc05 K split {split} tile_m={tile_m} fp32")
        _, _, y2, _ = run_ec(L, 330, tile_m, split=split, y_dtype=torch.float32)
        assert torch.equal(y1, y2)


@pytest.mark.parametrize("split", [4, 8])
def test_tc05_k_split_model_down_sampled(split):
    # The model's down projection (2048 x 8192) at 256 tokens, where the unsplit grid has 32 CTAs.
    L = config_layers(4, M=256, layers=(0,))[3]       # layer 0 carries a rank-32 compensator
    rows = np.array([0, 1, 127, 128, 255])
    got, ref, _, ws = run_ec(L, 256, 128, rows=rows, split=split)
    check_close(got, ref, True, f"tc05 K split {split} model down")
    assert int(ws[: (128 + 1024) * 1024].count_nonzero().item()) == 0, "EC flags not re-armed"
