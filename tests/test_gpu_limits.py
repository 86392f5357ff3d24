"""The largest batch the library takes (M = 65536 tokens) on every path, against the oracle at
sampled rows (the first and last tokens of the first, a middle and the last token blocks)."""
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

M_MAX = 65536
ROWS = np.array([0, 1, 127, 128, 32767, 32768, 65535])


@pytest.fixture(scope="module")
def layer():
    return make_layer("maxm", 777, M_MAX, 256, 256, 16, outlier_frac=0.02, outlier_scale=10.0, b_g=0.2)


def _ec(L):
    return spear.EC(to_dev_bf16(L.A_bits), to_dev_bf16(L.B_bits), to_dev_bf16(L.wg_bits), L.b_g)


@pytest.mark.parametrize("path", ["decode", "tc05", "tc05_256", "semifused"])
def test_max_tokens(layer, path):
    L = layer
    packed, scale, zero = spear.spear_pack_w4(to_dev(L.W))
    if path == "decode":
        plan = spear.spear_gemm_plan(16, L.N, L.K, L.rank)
        assert plan.kernel_id == spear.SPEAR_KERNEL_SPLITK
    else:
        plan = spear.spear_gemm_plan(M_MAX, L.N, L.K, L.rank)
        plan.kernel_id, plan.tile_n, plan.split_k = spear.SPEAR_KERNEL_TC05, 128, 1
        plan.tile_m = 256 if path == "tc05_256" else 128
        plan.flags = spear.SPEAR_PLAN_SEPARATE_EC if path == "semifused" else 0
    spear.spear_plan_update(plan, M_MAX, L.N, L.K, L.rank)
    ws = spear.alloc_workspace(plan.workspace_bytes)
    y = spear.spear_w4ec_gemm(to_dev_bf16(L.x(M_MAX)), packed, scale, zero, _ec(L), plan=plan, workspace=ws)
    torch.cuda.synchronize()
    assert spear.spear_get_device_status(ws) == 0
    p, s, z = oracle.pack_w4(L.W)
    ref = oracle.w4ec_gemm(L.x(M_MAX)[ROWS], p, s, z, L.A_bits, L.B_bits, L.wg_bits, L.b_g)
    check_close(host_f64(y[torch.from_numpy(ROWS).cuda()]), ref, True, f"M=65536 {path}")


def test_max_tokens_grouped(layer):
    L = layer
    packed, scale, zero = spear.spear_pack_w4_grouped(to_dev(L.W), 128)
    ws = spear.alloc_workspace(spear.spear_grouped_workspace_bytes(M_MAX, L.N, L.K, 128, L.rank))
    y = spear.spear_w4ec_gemm_grouped(to_dev_bf16(L.x(M_MAX)), packed, scale, zero, 128, _ec(L), workspace=ws)
    torch.cuda.synchronize()
    assert spear.spear_get_device_status(ws) == 0
    p, s, z = oracle.pack_w4_grouped(L.W, 128)
    ref = oracle.w4ec_gemm_grouped(L.x(M_MAX)[ROWS], p, s, z, 128, L.A_bits, L.B_bits, L.wg_bits, L.b_g)
    check_close(host_f64(y[torch.from_numpy(ROWS).cuda()]), ref, True, "M=65536 grouped")


def test_more_than_max_tokens_is_refused(layer):
    L = layer
    assert spear._lib.spear_gemm_plan(M_MAX + 1, L.N, L.K, L.rank, -1, spear.ctypes.byref(spear.spear_plan())) == 2
