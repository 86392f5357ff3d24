"""spear_w4ec_gemm_noalloc: the decode-sized layer for callers that cannot allocate device memory.

The entry point keeps its scratch in a library-owned device array instead of a caller
workspace.  Called twice in a row through the C ABI, it must give what the workspace entry point
gives, within the tolerance the parity tests use.  This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

from synthetic import config_layers
from gpu_helpers import check_close, host_f64, to_dev, to_dev_bf16

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import w4_gemm_error_channel_b200 as spear
else:
    spear = None


def _noalloc(lib, x, packed, scale, zero, ec, y, stream):
    P = ctypes.c_void_p
    M, K = x.shape
    N = packed.shape[0]
    ec_ref = ctypes.byref(ec.as_c()) if ec is not None else None
    return lib.spear_w4ec_gemm_noalloc(None, P(x.data_ptr()), M, N, K, P(packed.data_ptr()), P(scale.data_ptr()),
                                       P(zero.data_ptr()), ec_ref, P(y.data_ptr()), 0, P(stream.cuda_stream))


@pytest.mark.parametrize("M", [1, 16, 64])
@pytest.mark.parametrize("with_ec", [True, False])
def test_noalloc_matches_workspace_entry_point(M, with_ec):
    lib = spear._lib                                   # the C ABI, called directly
    L = config_layers(1, M=64)[0]                      # 4096 x 4096, rank 64
    packed, scale, zero = spear.spear_pack_w4(to_dev(L.W))
    ec = spear.EC(to_dev_bf16(L.A_bits), to_dev_bf16(L.B_bits), to_dev_bf16(L.wg_bits), L.b_g) if with_ec else None
    x = to_dev_bf16(L.x(M))
    stream = torch.cuda.current_stream()
    y_ref = spear.spear_w4ec_gemm(x, packed, scale, zero, ec)
    for call in range(2):                              # the scratch is reused by the second call
        y = torch.full((M, L.N), float("nan"), dtype=torch.bfloat16, device="cuda")
        assert _noalloc(lib, x, packed, scale, zero, ec, y, stream) == spear.SPEAR_OK
        torch.cuda.synchronize()
        check_close(host_f64(y), host_f64(y_ref), True, f"noalloc call {call} M={M} ec={with_ec}")


def test_noalloc_rejects_batches_beyond_its_scratch():
    L = config_layers(0)[0]
    packed, scale, zero = spear.spear_pack_w4(to_dev(L.W))
    x = torch.zeros((65, L.K), dtype=torch.bfloat16, device="cuda")
    y = torch.empty((65, L.N), dtype=torch.bfloat16, device="cuda")
    st = _noalloc(spear._lib, x, packed, scale, zero, None, y, torch.cuda.current_stream())
    assert st == 2                                     # SPEAR_ERR_UNSUPPORTED_SHAPE
