"""CUDA path against the CPU oracle, through the C ABI (python binding = argument marshalling).

Packing and unpacking are compared bit for bit.  The GEMM is compared within the
tolerance of tests/gpu_helpers.py: fully where the oracle finishes in seconds, and on
whole sampled token rows at the full workload sizes (token rows are independent, which
the oracle's own pins check).
"""
import functools

import numpy as np
import pytest
import torch

import oracle
from synthetic import bf16_bits_from_f32, config_layers, f32_from_bf16_bits, make_layer
from gpu_helpers import check_close, f16_bits, host_f64, to_dev, to_dev_bf16

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import w4_gemm_error_channel_b200 as spear
else:  # collected on CPU hosts only to be deselected by the gpu marker
    spear = None


@functools.lru_cache(maxsize=None)
def layer(idx, M=None, li=0, layers=None):
    return config_layers(idx, M=M, layers=layers)[li]


class Dev:
    """A layer's tensors on the device, packed by the CUDA packer."""

    def __init__(self, L, ec=True):
        self.L = L
        self.W = to_dev(L.W)
        self.packed, self.scale, self.zero = spear.spear_pack_w4(self.W)
        self.ec = None
        if ec and L.rank > 0:
            self.ec = spear.EC(to_dev_bf16(L.A_bits), to_dev_bf16(L.B_bits), to_dev_bf16(L.wg_bits), L.b_g)

    def run(self, M, y_dtype=torch.bfloat16, plan=None, ec="same", workspace=None, rows=None):
        x = to_dev_bf16(self.L.x(M))
        e = self.ec if ec == "same" else ec
        return spear.spear_w4ec_gemm(x, self.packed, self.scale, self.zero, e, y_dtype=y_dtype, plan=plan,
                                     workspace=workspace)

    def oracle_y(self, M, rows=None, ec=True):
        L = self.L
        x = L.x(M) if rows is None else L.x(M)[rows]
        p, s, z = oracle.pack_w4(L.W)
        if ec and L.rank > 0:
            return oracle.w4ec_gemm(x, p, s, z, L.A_bits, L.B_bits, L.wg_bits, L.b_g)
        return oracle.w4ec_gemm(x, p, s, z)


@functools.lru_cache(maxsize=None)
def dev_layer(idx, li=0, layers=None):
    return Dev(layer(idx, li=li, layers=layers))


# ----------------------------------------------------------------------------- packing

@pytest.mark.parametrize("idx", [0, 1, 2, 3])
def test_pack_bit_exact(idx):
    d = dev_layer(idx)
    p, s, z = oracle.pack_w4(d.L.W)
    assert np.array_equal(d.packed.cpu().numpy(), p)
    assert np.array_equal(f16_bits(d.scale), s)
    assert np.array_equal(f16_bits(d.zero), z)


def test_pack_edge_rows_and_bf16_input():
    rng = np.random.default_rng(3)
    N, K = 256, 320
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    W[0] = 0.0                                   # all-zero row
    W[1] = 1e-9                                  # scale underflows binary16
    W[2] = np.abs(W[2])                          # lo = 0
    W[3] = -np.abs(W[3])                         # hi = 0
    W[4] *= 1e4                                  # large range
    W[5, :] = 0.0
    W[5, 7] = 3.0                                # one spike
    q = rng.integers(0, 16, (8, K))
    q[:, 0], q[:, 1] = 0, 15
    W[8:16] = ((q - 7) * 0.0078125).astype(np.float32)   # on the int4 grid
    for Wt in (W, f32_from_bf16_bits(bf16_bits_from_f32(W))):
        dev = to_dev(Wt) if Wt is W else to_dev_bf16(bf16_bits_from_f32(W))
        packed, scale, zero = spear.spear_pack_w4(dev)
        p, s, z = oracle.pack_w4(Wt)
        assert np.array_equal(packed.cpu().numpy(), p)
        assert np.array_equal(f16_bits(scale), s)
        assert np.array_equal(f16_bits(zero), z)


@pytest.mark.parametrize("K", [2, 6, 14, 64, 130])
def test_pack_odd_row_lengths(K):
    rng = np.random.default_rng(K)
    W = (rng.standard_normal((37, K)) * 0.05).astype(np.float32)
    packed, scale, zero = spear.spear_pack_w4(to_dev(W))
    p, s, z = oracle.pack_w4(W)
    assert np.array_equal(packed.cpu().numpy(), p)
    assert np.array_equal(f16_bits(scale), s) and np.array_equal(f16_bits(zero), z)
    q, qz = spear.spear_debug_unpack_w4(packed, zero, K)
    assert np.array_equal(q.cpu().numpy(), oracle.unpack_nibbles(p, K))


@pytest.mark.parametrize("idx", [0, 1])
def test_unpack_exact(idx):
    d = dev_layer(idx)
    K = d.L.K
    q, qz = spear.spear_debug_unpack_w4(d.packed, d.zero, K)
    p, s, z = oracle.pack_w4(d.L.W)
    q_ref = oracle.unpack_nibbles(p, K)
    assert np.array_equal(q.cpu().numpy(), q_ref)
    z_ref = z.view(np.float16).astype(np.float64)
    assert np.array_equal(qz.float().cpu().numpy().astype(np.float64), q_ref.astype(np.float64) - z_ref[:, None])


# ----------------------------------------------------------------------------- GEMM

def test_tiny_full_bf16_and_fp32():
    d = dev_layer(0)
    ref = d.oracle_y(4)
    check_close(host_f64(d.run(4)), ref, True, "tiny bf16")
    check_close(host_f64(d.run(4, y_dtype=torch.float32)), ref, False, "tiny fp32")


@pytest.mark.parametrize("M", [1, 4, 16])
def test_decode_qo(M):
    d = dev_layer(1)
    ref = d.oracle_y(M)
    check_close(host_f64(d.run(M)), ref, True, f"decode-qo M={M}")
    check_close(host_f64(d.run(M, y_dtype=torch.float32)), ref, False, f"decode-qo M={M} fp32")


@pytest.mark.parametrize("M", [1, 8, 32, 64])
def test_decode_mlp(M):
    d = dev_layer(2)
    rows = np.arange(M) if M <= 8 else np.array([0, 3, M // 2, M - 1])
    ref = d.oracle_y(M, rows=rows)
    check_close(host_f64(d.run(M))[rows], ref, True, f"decode-mlp M={M}")


def test_prefill_sampled_rows():
    d = dev_layer(3)
    M = 2048
    rows = np.array([0, 1, 127, 128, 1000, 2047])
    ref = d.oracle_y(M, rows=rows)
    y = host_f64(d.run(M))
    check_close(y[rows], ref, True, "prefill")
    assert np.isfinite(y).all()


@pytest.mark.parametrize("li", [0, 1, 2, 3])
@pytest.mark.parametrize("layer_idx", [0, 2])  # layer 0 carries an EC, layer 2 does not
def test_sweep_layers(layer_idx, li):
    d = dev_layer(4, li=li, layers=(layer_idx,))
    for M in (1, 16, 256):
        rows = np.arange(M) if M <= 16 else np.array([0, 100, 255])
        ref = d.oracle_y(M, rows=rows)
        check_close(host_f64(d.run(M))[rows], ref, True, f"sweep L{layer_idx}.{li} M={M}")


@pytest.mark.parametrize("M", [1, 2, 3, 5, 7, 9, 15, 17, 31, 33, 63, 65, 100])
@pytest.mark.parametrize("r", [0, 16, 48])
def test_ragged_tokens_and_k_tail(M, r):
    # K = 320 is a multiple of 64 but not of 128: the last K window is half full.
    L = make_layer("ragged", 77 + r, 100, 256, 320, r, outlier_frac=0.02, outlier_scale=10.0)
    d = Dev(L)
    ref = d.oracle_y(M)
    check_close(host_f64(d.run(M)), ref, True, f"ragged M={M} r={r}")
    plan = spear.spear_gemm_plan(M, L.N, L.K, r)
    plan.split_k = 2                      # K slices of 192 and 128 codes: a half-full window
    plan.tile_n = 16
    ws = spear.alloc_workspace(1 << 24)
    check_close(host_f64(d.run(M, plan=plan, workspace=ws)), ref, True, f"ragged M={M} r={r} split 2")


def test_gate_off_is_bitwise_plain_and_deterministic():
    L = layer(1)
    d = dev_layer(1)
    off = spear.EC(d.ec.A, d.ec.B, d.ec.w_g, float("-inf"))
    for M in (1, 16):
        plan = spear.spear_gemm_plan(M, L.N, L.K, L.rank)
        y_plain = d.run(M, plan=plan, ec=None)
        y_off = d.run(M, plan=plan, ec=off)
        assert torch.equal(y_plain, y_off)
        y1 = d.run(M, plan=plan)
        y2 = d.run(M, plan=plan)
        assert torch.equal(y1, y2)


def test_split_k_variants_agree():
    d = dev_layer(1)
    L = d.L
    ref = d.oracle_y(16)
    for split in (1, 2, 4, 8):
        plan = spear.spear_gemm_plan(16, L.N, L.K, L.rank)
        plan.split_k = split
        k_slice = ((L.K + split - 1) // split + 63) // 64 * 64
        windows = (k_slice + 511) // 512          # 128-wide K windows per warp
        plan.tile_n = 16 * min(8, 8 // windows)   # compiled tilings keep windows * (tile_n / 16) <= 8
        plan.workspace_bytes = 0
        ws = spear.alloc_workspace(1 << 26)
        check_close(host_f64(d.run(16, plan=plan, workspace=ws)), ref, True, f"split {split}")


def test_shared_workspace_across_shapes():
    # Tickets re-arm themselves: one workspace serves a sequence of different problems.
    ws = spear.alloc_workspace(1 << 27)
    d1, d0 = dev_layer(1), dev_layer(0)
    for _ in range(2):
        for d, M in ((d1, 16), (d0, 4), (d1, 1), (d1, 4), (d0, 1)):
            check_close(host_f64(d.run(M, workspace=ws)), d.oracle_y(M), True, f"{d.L.name} M={M}")
    assert spear.spear_get_device_status(ws) == 0
    zeroed = ws[: (128 + 1024) * 1024].cpu()      # control block + EC accumulators
    assert int(zeroed.count_nonzero()) == 0, "counters or accumulators not re-armed"


def test_empty_batch():
    d = dev_layer(0)
    x = torch.empty((0, d.L.K), dtype=torch.bfloat16, device="cuda")
    y = spear.spear_w4ec_gemm(x, d.packed, d.scale, d.zero, d.ec)
    assert y.shape == (0, d.L.N)


# ----------------------------------------------------------------------------- prepared layer

def test_prepared_layer_matches_call():
    # W4ECLayer binds the weights once; its calls equal spear_w4ec_gemm's bit for bit.
    d = dev_layer(1)
    lay = spear.W4ECLayer(d.packed, d.scale, d.zero, d.ec)
    stream = torch.cuda.Stream()
    for M in (1, 4, 16, 1):
        x = to_dev_bf16(d.L.x(M))
        y = torch.empty((M, d.L.N), dtype=torch.bfloat16, device="cuda")
        lay(x, y=y, stream=stream)
        stream.synchronize()
        assert torch.equal(y, d.run(M))
    assert spear.spear_get_device_status(lay.workspace) == 0
    x = to_dev_bf16(d.L.x(4))
    with pytest.raises(ValueError):
        lay(x.cpu())                                              # activations on the host
    with pytest.raises(ValueError):
        lay(x, y=torch.empty((4, d.L.N), dtype=torch.float32, device="cuda"))   # wrong output dtype
    with pytest.raises(ValueError):
        lay(x[:, :128].contiguous())                              # wrong K


# ----------------------------------------------------------------------------- separate EC pass

@pytest.mark.parametrize("idx,M", [(1, 1), (1, 4), (1, 16), (2, 8), (0, 4)])
def test_separate_ec_pass(idx, M):
    # Plan flag SPEAR_PLAN_SEPARATE_EC: the weight-streaming CTAs write fp32 main terms and a second
    # kernel applies the compensator.  Twice in a row on one workspace (the accumulators re-arm).
    d = dev_layer(idx)
    L = d.L
    ref = d.oracle_y(M)
    plan = spear.spear_gemm_plan(M, L.N, L.K, L.rank)
    if plan.kernel_id != spear.SPEAR_KERNEL_SPLITK:
        pytest.skip("not a split-K decode plan")
    plan.flags = spear.SPEAR_PLAN_SEPARATE_EC
    ws = spear.alloc_workspace((1 << 21) + min(M, 256) * L.N * 4)
    for _ in range(2):
        check_close(host_f64(d.run(M, plan=plan, workspace=ws)), ref, True, f"separate EC {L.name} M={M}")
    assert spear.spear_get_device_status(ws) == 0
    assert int(ws[: (128 + 1024) * 1024].count_nonzero().item()) == 0, "accumulators not re-armed"


@pytest.mark.parametrize("M", [23, 300])
def test_separate_ec_pass_ragged(M):
    L = make_layer("sep", 71 + M, M, 384, 1024, 32, outlier_frac=0.01, outlier_scale=20.0, b_g=0.3)
    d = Dev(L)
    plan = spear.spear_gemm_plan(M, L.N, L.K, L.rank)
    plan.kernel_id, plan.tile_n, plan.split_k, plan.tile_m = spear.SPEAR_KERNEL_SPLITK, 32, 2, 16
    plan.flags = spear.SPEAR_PLAN_SEPARATE_EC
    ws = spear.alloc_workspace((1 << 21) + min(M, 256) * L.N * 4)
    check_close(host_f64(d.run(M, plan=plan, workspace=ws)), d.oracle_y(M), True, f"separate EC M={M}")
    assert spear.spear_get_device_status(ws) == 0
    assert int(ws[: (128 + 1024) * 1024].count_nonzero().item()) == 0


def test_separate_ec_pass_gate_off():
    # g = 0 exactly: the applied term adds zeros, so y equals the plain layer within the tolerance
    # and the fp32 debug output equals the fused kernel's plain result exactly.
    L = make_layer("sepg", 5, 8, 512, 1024, 64)
    d = Dev(L)
    plan = spear.spear_gemm_plan(8, L.N, L.K, L.rank)
    plan.flags = spear.SPEAR_PLAN_SEPARATE_EC
    ws = spear.alloc_workspace((1 << 21) + 8 * L.N * 4)
    ec_off = spear.EC(d.ec.A, d.ec.B, d.ec.w_g, float("-inf"))
    y_off = d.run(8, plan=plan, workspace=ws, ec=ec_off, y_dtype=torch.float32)
    plain_plan = spear.spear_plan.from_buffer_copy(plan)
    plain_plan.flags = 0
    y_plain = d.run(8, plan=plain_plan, workspace=spear.alloc_workspace(1 << 21), ec=None, y_dtype=torch.float32)
    assert torch.equal(y_off, y_plain)
