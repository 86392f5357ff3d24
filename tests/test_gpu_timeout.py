"""Bounded waits give up with an error status, and the context stays usable.

The fused decode kernels wait for the compensator's accumulators: every int64 word counts, in its
low 8 bits, the K slices added to it, and a reader waits (for about a second at most) until the
count equals the number of slices.  Here the accumulator area of the workspace starts with count
128 in every word instead of 0, so no word ever reaches the slice count (128 + S is never S
modulo 256): the wait runs out, the kernel records it in the workspace's error word and returns,
and spear_get_device_status reports SPEAR_ERR_TIMEOUT.  Nothing faults or hangs: the next call on
a re-zeroed workspace gives the right result.
"""
import numpy as np
import pytest
import torch

import oracle
from synthetic import config_layers
from gpu_helpers import check_close, host_f64, to_dev, to_dev_bf16

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import w4_gemm_error_channel_b200 as spear
else:
    spear = None

CTRL_BYTES, TACC_BYTES = 128 * 1024, 1024 * 1024


def _layer():
    L = config_layers(0)[0]                       # 512 x 512, rank 16: one wave of CTAs
    packed, scale, zero = spear.spear_pack_w4(to_dev(L.W))
    ec = spear.EC(to_dev_bf16(L.A_bits), to_dev_bf16(L.B_bits), to_dev_bf16(L.wg_bits), L.b_g)
    return L, packed, scale, zero, ec


def _poison(ws):
    words = ws[CTRL_BYTES:CTRL_BYTES + TACC_BYTES].view(torch.int64)
    words.fill_(0x80)                             # count 128, value 0
    torch.cuda.synchronize()


@pytest.mark.parametrize("kernel", ["split-K decode", "stream-K register path"])
def test_accumulator_wait_gives_up_with_timeout_status(kernel):
    L, packed, scale, zero, ec = _layer()
    M = 4
    x = to_dev_bf16(L.x(M))
    codes = packed
    if kernel == "split-K decode":
        plan = spear.spear_gemm_plan(M, L.N, L.K, L.rank)
        plan.kernel_id, plan.tile_n, plan.split_k, plan.tile_m, plan.flags = 1, 32, 1, 8, 0
        spear.spear_plan_update(plan, M, L.N, L.K, L.rank)
    else:
        plan = spear.spear_gemm_plan_tiled(M, L.N, L.K, L.rank)
        codes = spear.spear_tile_w4(packed)
    ws = spear.alloc_workspace(plan.workspace_bytes)
    _poison(ws)
    y = spear.spear_w4ec_gemm(x, codes, scale, zero, ec, plan=plan, workspace=ws)
    torch.cuda.synchronize()                      # the kernel returned: no hang, no fault
    assert int(ws[:4].view(torch.int32).item()) != 0           # the error word records the give-up
    assert spear.spear_get_device_status(ws, clear=False) == spear.SPEAR_ERR_TIMEOUT
    # Still usable: a re-zeroed workspace gives the layer's result again.
    ws.zero_()
    y = spear.spear_w4ec_gemm(x, codes, scale, zero, ec, plan=plan, workspace=ws)
    torch.cuda.synchronize()
    assert spear.spear_get_device_status(ws) == spear.SPEAR_OK
    p, s, z = oracle.pack_w4(L.W)
    ref = oracle.w4ec_gemm(L.x(M), p, s, z, L.A_bits, L.B_bits, L.wg_bits, L.b_g)
    check_close(host_f64(y), ref, True, f"after timeout, {kernel}")
