"""spear_w4ec_gemm_noalloc: the decode-sized layer for callers that cannot allocate device memory.

Some callers own no device allocator of their own (an engine whose memory belongs to another
framework that hands out no scratch buffers) or must not allocate on a latency-critical path.  For
them the entry point keeps its scratch in a library-owned device array instead of a caller
workspace.  Called twice in a row through the C ABI it must give exactly what the workspace entry
point gives with the same plan (both run the same deterministic kernel), and match the oracle.
This file is collected last on purpose.
"""
import ctypes

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

SPEAR_ERR_INVALID_ARG, SPEAR_ERR_UNSUPPORTED_SHAPE = 1, 2


def _noalloc(x, packed, scale, zero, ec, y, plan=None):
    """The C call itself (no Python-side allocation)."""
    P = ctypes.c_void_p
    M, K = x.shape
    N = packed.shape[0]
    ec_ref = ctypes.byref(ec.as_c()) if ec is not None else None
    plan_ref = ctypes.byref(plan) if plan is not None else None
    yd = spear.SPEAR_FP32 if y.dtype == torch.float32 else spear.SPEAR_BF16
    stream = torch.cuda.current_stream()
    return spear._lib.spear_w4ec_gemm_noalloc(plan_ref, P(x.data_ptr()), M, N, K, P(packed.data_ptr()),
                                              P(scale.data_ptr()), P(zero.data_ptr()), ec_ref, P(y.data_ptr()), yd,
                                              P(stream.cuda_stream))


def _split_k_plan(M, N, K, rank):
    """The split-K decode plan the entry point runs: the dispatcher's when it is one, else a fixed one."""
    p = spear.spear_gemm_plan(M, N, K, rank)
    if p.kernel_id != spear.SPEAR_KERNEL_SPLITK or p.flags != 0:
        p.kernel_id, p.tile_n, p.split_k, p.flags = spear.SPEAR_KERNEL_SPLITK, 32, 4, 0
        p.tile_m = 8 if M <= 8 else (16 if M <= 16 else 32)
    return spear.spear_plan_update(p, M, N, K, rank)


def _layer(kind, M):
    if kind == "qo":                                   # 4096 x 4096, rank 64
        return config_layers(1, M=M)[0]
    if kind == "mlp":                                  # 22016 x 4096, rank 64
        return config_layers(2, M=M)[0]
    # rank 256 (the largest the scratch holds, at 64 tokens)
    return make_layer("noalloc-r256", 4242, M, 1024, 2048, 256, outlier_frac=0.01, outlier_scale=20.0, b_g=0.5)


@pytest.mark.parametrize("kind,M,with_ec,fp32", [
    ("qo", 1, True, False), ("qo", 16, True, False), ("qo", 64, True, False), ("qo", 16, False, False),
    ("qo", 16, True, True), ("mlp", 64, True, False), ("r256", 64, True, False), ("r256", 64, True, True),
])
def test_noalloc_matches_workspace_entry_point(kind, M, with_ec, fp32):
    L = _layer(kind, M)
    packed, scale, zero = spear.spear_pack_w4(to_dev(L.W))
    ec = spear.EC(to_dev_bf16(L.A_bits), to_dev_bf16(L.B_bits), to_dev_bf16(L.wg_bits), L.b_g) if with_ec else None
    x = to_dev_bf16(L.x(M))
    y_dtype = torch.float32 if fp32 else torch.bfloat16
    rank = L.rank if with_ec else 0
    plan = _split_k_plan(M, L.N, L.K, rank)
    y_ref = spear.spear_w4ec_gemm(x, packed, scale, zero, ec, y_dtype=y_dtype, plan=plan)
    rows = np.arange(M) if M <= 16 else np.array([0, 1, M // 2, M - 1])
    p, s, z = oracle.pack_w4(L.W)
    xr = L.x(M)[rows]
    ref = oracle.w4ec_gemm(xr, p, s, z, L.A_bits, L.B_bits, L.wg_bits, L.b_g) if with_ec else \
        oracle.w4ec_gemm(xr, p, s, z)
    # The explicit plan, then the entry point's own (plan = NULL), each twice in a row: the array
    # keeps the previous call's contents, which the kernel re-arms.
    first_null = None
    for call, pl in enumerate((plan, plan, None, None)):
        y = torch.full((M, L.N), float("nan"), dtype=y_dtype, device="cuda")
        assert _noalloc(x, packed, scale, zero, ec, y, pl) == spear.SPEAR_OK
        torch.cuda.synchronize()
        if pl is not None:
            assert torch.equal(y, y_ref), f"noalloc call {call} {kind} M={M} differs from spear_w4ec_gemm"
        elif first_null is None:
            first_null = y
        else:
            assert torch.equal(y, first_null), f"noalloc call {call} {kind} M={M} is not deterministic"
        check_close(host_f64(y)[rows], ref, not fp32, f"noalloc call {call} {kind} M={M}")
    assert spear.spear_noalloc_get_device_status(clear=False) == spear.SPEAR_OK


def test_noalloc_python_wrapper_allocates_nothing_and_needs_y():
    L = _layer("qo", 4)
    packed, scale, zero = spear.spear_pack_w4(to_dev(L.W))
    ec = spear.EC(to_dev_bf16(L.A_bits), to_dev_bf16(L.B_bits), to_dev_bf16(L.wg_bits), L.b_g)
    x = to_dev_bf16(L.x(4))
    y = torch.empty((4, L.N), dtype=torch.bfloat16, device="cuda")
    out = spear.spear_w4ec_gemm_noalloc(x, packed, scale, zero, y, ec)
    assert out is y
    torch.cuda.synchronize()
    check_close(host_f64(y), oracle.w4ec_gemm(L.x(4), *oracle.pack_w4(L.W), L.A_bits, L.B_bits, L.wg_bits, L.b_g),
                True, "wrapper")
    with pytest.raises(TypeError):
        spear.spear_w4ec_gemm_noalloc(x, packed, scale, zero)           # y is required


def test_noalloc_rejects_what_it_cannot_run():
    L = config_layers(0)[0]
    packed, scale, zero = spear.spear_pack_w4(to_dev(L.W))
    x = torch.zeros((65, L.K), dtype=torch.bfloat16, device="cuda")
    y = torch.empty((65, L.N), dtype=torch.bfloat16, device="cuda")
    assert _noalloc(x, packed, scale, zero, None, y) == SPEAR_ERR_UNSUPPORTED_SHAPE   # beyond its 64 tokens
    x, y = x[:16].contiguous(), y[:16].contiguous()
    tc = spear.spear_gemm_plan(16, L.N, L.K, 0)
    tc.kernel_id, tc.tile_n, tc.split_k, tc.tile_m, tc.flags = spear.SPEAR_KERNEL_TC05, 128, 1, 128, 0
    assert _noalloc(x, packed, scale, zero, None, y, tc) == SPEAR_ERR_INVALID_ARG      # needs a workspace
    st = spear.spear_gemm_plan(16, L.N, L.K, 0)
    st.kernel_id, st.tile_n, st.split_k, st.tile_m, st.flags = spear.SPEAR_KERNEL_STREAM, 128, 64, 16, 0
    assert _noalloc(x, packed, scale, zero, None, y, st) == SPEAR_ERR_INVALID_ARG
    sep = _split_k_plan(16, L.N, L.K, L.rank)
    sep.flags = spear.SPEAR_PLAN_SEPARATE_EC
    ec = spear.EC(to_dev_bf16(L.A_bits), to_dev_bf16(L.B_bits), to_dev_bf16(L.wg_bits), L.b_g)
    assert _noalloc(x, packed, scale, zero, ec, y, sep) == SPEAR_ERR_INVALID_ARG
