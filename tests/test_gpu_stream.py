"""The small-batch stream-K kernels (SPEAR_KERNEL_STREAM, and SPEAR_KERNEL_STREAM_RK on codes in the
tile order of spear_tile_w4) against the CPU oracle, through the C ABI.

Every token tile (8 to 64), pipeline-stage width (128, 256 codes) and ring mode (two CTAs per SM,
or one with a deep ring) is run with explicit plans; the tolerance is the one of
tests/gpu_helpers.py.  The tiles that straddle CTAs meet in a fixed order, so repeated calls are
bit-identical, and a compensator whose gate is exactly 0 gives the plain layer bit for bit.
"""
import functools

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

ZEROED = (128 + 1024) * 1024          # control block + EC accumulators: zero at rest


KERNELS = ["tc", "rk"]                 # tcgen05 (converted weights in TMEM) and register (mma.sync) paths


def stream_plan(M, N, K, rank, bn, kc, deep, kernel="tc"):
    p = spear.spear_plan()
    kid = spear.SPEAR_KERNEL_STREAM if kernel == "tc" else spear.SPEAR_KERNEL_STREAM_RK
    p.kernel_id, p.tile_n, p.tile_m, p.split_k = kid, 128, bn, kc
    p.flags = (spear.SPEAR_PLAN_DEEP_RING if deep else 0) | (spear.SPEAR_PLAN_W4_TILES if kernel == "rk" else 0)
    return spear.spear_plan_update(p, M, N, K, rank)


class Dev:
    def __init__(self, L):
        self.L = L
        self.packed, self.scale, self.zero = spear.spear_pack_w4(to_dev(L.W))
        self._tiled = None
        self.ec = None
        if L.rank > 0:
            self.ec = spear.EC(to_dev_bf16(L.A_bits), to_dev_bf16(L.B_bits), to_dev_bf16(L.wg_bits), L.b_g)
        self.xd = {}

    def x(self, M):
        if M not in self.xd:
            self.xd[M] = to_dev_bf16(self.L.x(M))
        return self.xd[M]

    @property
    def tiled(self):
        if self._tiled is None:
            self._tiled = spear.spear_tile_w4(self.packed)
        return self._tiled

    def run(self, M, plan, ws, y_dtype=torch.bfloat16, ec="same", y=None, stream=None):
        e = self.ec if ec == "same" else ec
        codes = self.tiled if plan is not None and plan.flags & spear.SPEAR_PLAN_W4_TILES else self.packed
        return spear.spear_w4ec_gemm(self.x(M), codes, self.scale, self.zero, e, y=y, y_dtype=y_dtype,
                                     plan=plan, workspace=ws, stream=stream)

    def ref(self, M, rows=None, ec=True):
        L = self.L
        x = L.x(M) if rows is None else L.x(M)[rows]
        p, s, z = oracle.pack_w4(L.W)
        if ec and L.rank > 0:
            return oracle.w4ec_gemm(x, p, s, z, L.A_bits, L.B_bits, L.wg_bits, L.b_g)
        return oracle.w4ec_gemm(x, p, s, z)


@functools.lru_cache(maxsize=None)
def dev(idx, li=0, layer=None):
    layers = (layer,) if layer is not None else None
    return Dev(config_layers(idx, layers=layers)[li])


def tilings(M, K, ec_rank, kernel="tc"):
    out = []
    for bn in ((16, 32, 64) if kernel == "tc" else (8, 16, 32, 64)):
        if M > bn:
            continue
        for kc in (128, 256):
            if K % kc:
                continue
            for deep in (False, True):
                out.append((bn, kc, deep))
    return out


def ok_status(ws):
    assert spear.spear_get_device_status(ws) == 0, "a bounded wait timed out"
    assert int(ws[:ZEROED].count_nonzero().item()) == 0, "control words or accumulators not re-armed"


def _configurable(M, L, bn, kc, deep, kernel="tc"):
    try:
        return stream_plan(M, L.N, L.K, L.rank, bn, kc, deep, kernel)
    except spear.SpearError:
        return None


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("M", [1, 4])
def test_tiny_every_tiling(M, kernel):
    d = dev(0)
    L = d.L
    ref = d.ref(M)
    ref_plain = d.ref(M, ec=False)
    for bn, kc, deep in tilings(M, L.K, L.rank, kernel):
        plan = _configurable(M, L, bn, kc, deep, kernel)
        if plan is None:
            continue
        ws = spear.alloc_workspace(plan.workspace_bytes)
        what = f"tiny {kernel} M={M} bn={bn} kc={kc} deep={deep}"
        check_close(host_f64(d.run(M, plan, ws)), ref, True, what)
        check_close(host_f64(d.run(M, plan, ws, y_dtype=torch.float32)), ref, False, what + " fp32")
        plain = stream_plan(M, L.N, L.K, 0, bn, kc, deep, kernel)
        check_close(host_f64(d.run(M, plain, ws, ec=None)), ref_plain, True, what + " no EC")
        ok_status(ws)


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("M", [1, 4, 16])
def test_decode_qo(M, kernel):
    d = dev(1)
    L = d.L
    ref = d.ref(M)
    tiles = [(16, 128, False), (16, 256, False), (16, 256, True), (32, 128, False), (64, 128, True)]
    if kernel == "rk":
        tiles += [(8, 128, False), (8, 256, False), (8, 256, True)]
    for bn, kc, deep in tiles:
        if M > bn:
            continue
        plan = stream_plan(M, L.N, L.K, L.rank, bn, kc, deep, kernel)
        ws = spear.alloc_workspace(plan.workspace_bytes)
        what = f"decode-qo {kernel} M={M} bn={bn} kc={kc} deep={deep}"
        check_close(host_f64(d.run(M, plan, ws)), ref, True, what)
        check_close(host_f64(d.run(M, plan, ws, y_dtype=torch.float32)), ref, False, what + " fp32")
        ok_status(ws)


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("M", [1, 8, 32, 64])
def test_decode_mlp_sampled_rows(M, kernel):
    d = dev(2)
    L = d.L
    rows = np.arange(M) if M <= 8 else np.array([0, 3, M // 2, M - 1])
    ref = d.ref(M, rows=rows)
    bn = (8 if kernel == "rk" and M <= 8 else 16) if M <= 16 else (32 if M <= 32 else 64)
    for kc, deep in [(256, True), (128, False), (128, True)]:
        plan = _configurable(M, L, bn, kc, deep, kernel)
        if plan is None:
            continue
        ws = spear.alloc_workspace(plan.workspace_bytes)
        y = host_f64(d.run(M, plan, ws))
        check_close(y[rows], ref, True, f"decode-mlp {kernel} M={M} kc={kc} deep={deep}")
        assert np.isfinite(y).all()
        ok_status(ws)


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("li", [0, 1, 2, 3])
@pytest.mark.parametrize("layer", [0, 2])           # layer 0 carries a compensator, layer 2 does not
def test_sweep_linears(layer, li, kernel):
    d = dev(4, li=li, layer=layer)
    L = d.L
    for M in (1, 16):
        ref = d.ref(M)
        plan = stream_plan(M, L.N, L.K, L.rank, 16, 128, False, kernel)
        ws = spear.alloc_workspace(plan.workspace_bytes)
        check_close(host_f64(d.run(M, plan, ws)), ref, True, f"sweep {kernel} L{layer}.{li} M={M}")
        ok_status(ws)


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("M", [1, 2, 3, 7, 9, 15, 16, 17, 31, 33, 47, 63, 64])
@pytest.mark.parametrize("r", [0, 16, 48, 128, 256])
def test_ragged_shapes(M, r, kernel):
    # N = 384: three tiles; K = 640 = 5 stages of 128 codes, so tiles straddle CTAs unevenly.
    L = make_layer("stream-ragged", 91 + r, 64, 384, 640, r, outlier_frac=0.02, outlier_scale=10.0, b_g=0.5)
    d = Dev(L)
    ref = d.ref(M)
    bn = (8 if kernel == "rk" and M <= 8 else 16) if M <= 16 else (32 if M <= 32 else 64)
    for deep in (False, True):
        plan = _configurable(M, L, bn, 128, deep, kernel)
        if plan is None:
            continue
        ws = spear.alloc_workspace(plan.workspace_bytes)
        check_close(host_f64(d.run(M, plan, ws)), ref, True, f"ragged {kernel} M={M} r={r} deep={deep}")
        ok_status(ws)


@pytest.mark.parametrize("kernel", KERNELS)
def test_gate_off_is_bitwise_plain_and_deterministic(kernel):
    d = dev(1)
    L = d.L
    off = spear.EC(d.ec.A, d.ec.B, d.ec.w_g, float("-inf"))
    for M, bn, kc in ((1, 16, 128), (16, 16, 256), (16, 32, 128)):
        plan = stream_plan(M, L.N, L.K, L.rank, bn, kc, False, kernel)
        plain = stream_plan(M, L.N, L.K, 0, bn, kc, False, kernel)
        ws = spear.alloc_workspace(plan.workspace_bytes)
        y_plain = d.run(M, plain, ws, ec=None, y_dtype=torch.float32)
        y_off = d.run(M, plan, ws, ec=off, y_dtype=torch.float32)
        assert torch.equal(y_plain, y_off)
        y1, y2 = d.run(M, plan, ws), d.run(M, plan, ws)
        assert torch.equal(y1, y2)
        ok_status(ws)


@pytest.mark.parametrize("kernel", KERNELS)
def test_chained_calls_in_one_stream(kernel):
    # Back-to-back calls on one stream overlap through programmatic dependent launch: each call's
    # weight stream starts while the previous one finishes.  Alternate two layers and two batch
    # sizes on one workspace, then check every output.
    d1, d0 = dev(1), dev(0)
    stream = torch.cuda.Stream()
    plans = {}
    for d in (d1, d0):
        for M in (1, 16):
            # decode-qo: 64-code stages with the deep ring at M = 1 (a small CTA that must still hold
            # its SM alone), 128-code stages with two CTAs per SM at M = 16
            deep = d is d1 and M == 1
            plans[(d.L.name, M)] = stream_plan(M, d.L.N, d.L.K, d.L.rank, 16, 128 if (d is d0 or deep) else 256, deep,
                                               kernel)
    ws = spear.alloc_workspace(max(p.workspace_bytes for p in plans.values()))
    seq = [(d1, 16), (d1, 16), (d0, 1), (d1, 1), (d0, 16), (d1, 16)] * 3
    outs = []
    with torch.cuda.stream(stream):
        for d, M in seq:
            outs.append(d.run(M, plans[(d.L.name, M)], ws, stream=stream))
    stream.synchronize()
    refs = {}
    for (d, M), y in zip(seq, outs):
        key = (d.L.name, M)
        if key not in refs:
            refs[key] = d.ref(M)
        check_close(host_f64(y), refs[key], True, f"chained {key}")
    ok_status(ws)


@pytest.mark.parametrize("kernel", KERNELS)
def test_graph_replay(kernel):
    d = dev(1)
    L = d.L
    plan = stream_plan(16, L.N, L.K, L.rank, 16, 128, False, kernel)
    ws = spear.alloc_workspace(plan.workspace_bytes)
    x = d.x(16)
    y = torch.empty((16, L.N), dtype=torch.bfloat16, device="cuda")
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        d.run(16, plan, ws, y=y, stream=stream)          # warm-up outside the capture
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for _ in range(4):
            spear.spear_w4ec_gemm(x, d.tiled if kernel == "rk" else d.packed, d.scale, d.zero, d.ec, y=y, plan=plan,
                                  workspace=ws, stream=stream)
    y.zero_()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    check_close(host_f64(y), d.ref(16), True, "graph replay")
    ok_status(ws)


def test_rejects_bad_stream_plans():
    d = dev(0)
    L = d.L
    plan = stream_plan(4, L.N, L.K, L.rank, 16, 128, False)
    bad = spear.spear_plan.from_buffer_copy(plan)
    bad.tile_m = 8                                       # not a token tile of this kernel
    with pytest.raises(spear.SpearError):
        spear.spear_plan_update(bad, 4, L.N, L.K, L.rank)
    bad = spear.spear_plan.from_buffer_copy(plan)
    bad.split_k = 64                                     # one sub-chunk per stage: not taken
    with pytest.raises(spear.SpearError):
        spear.spear_plan_update(bad, 4, L.N, L.K, L.rank)
    with pytest.raises(spear.SpearError):                # more tokens than the tile
        spear.spear_plan_update(spear.spear_plan.from_buffer_copy(plan), 17, L.N, L.K, L.rank)
    # The register path: 64 tokens only with the deep ring, ranks up to 128.
    with pytest.raises(spear.SpearError):
        stream_plan(64, L.N, L.K, L.rank, 64, 128, False, "rk")
    stream_plan(64, L.N, L.K, L.rank, 64, 128, True, "rk")
    with pytest.raises(spear.SpearError):
        stream_plan(4, L.N, L.K, 256, 8, 128, False, "rk")
    # Tile-order codes: required by the register path, refused by the others.
    rk = stream_plan(4, L.N, L.K, L.rank, 8, 128, False, "rk")
    bad = spear.spear_plan.from_buffer_copy(rk)
    bad.flags &= ~spear.SPEAR_PLAN_W4_TILES
    with pytest.raises(spear.SpearError):
        spear.spear_plan_update(bad, 4, L.N, L.K, L.rank)
    bad = spear.spear_plan.from_buffer_copy(plan)
    bad.flags |= spear.SPEAR_PLAN_W4_TILES
    with pytest.raises(spear.SpearError):
        spear.spear_plan_update(bad, 4, L.N, L.K, L.rank)
    H = 4
    mlp = spear.EC(d.ec.A, d.ec.B, d.ec.w_g, 0.0,
                   gate_w1=torch.zeros((H, L.rank), device="cuda"), gate_b1=torch.zeros(H, device="cuda"),
                   gate_w2=torch.zeros((L.rank, H), device="cuda"), gate_b2=torch.zeros(L.rank, device="cuda"))
    ws = spear.alloc_workspace(plan.workspace_bytes)
    with pytest.raises(spear.SpearError):               # the MLP gate is not taken by this kernel
        d.run(4, plan, ws, ec=mlp)


def _tile_order_numpy(packed, N, K):
    """The tile order restated on the host: 128 x 128-code blocks, row r's 64 bytes at r * 64,
    word 4c + w of a block row holding codes 8s .. 8s + 7 (s = 2c + w, or 8 + 2c + w - 2 for
    w >= 2), code 8s + j in nibble (j // 2) + 4 (j % 2)."""
    words = np.ascontiguousarray(packed).view(np.uint32).reshape(N, K // 8)
    src = [2 * (i // 4) + i % 4 if i % 4 < 2 else 8 + 2 * (i // 4) + i % 4 - 2 for i in range(16)]
    words = words.reshape(N, K // 128, 16)[:, :, src].reshape(N, K // 8)
    codes = np.stack([(words >> (4 * j)) & 0xF for j in range(8)], axis=-1)        # [N, K/8, 8]
    out_words = np.zeros_like(words)
    for j in range(8):
        out_words |= codes[..., j] << np.uint32(4 * (j // 2 + 4 * (j % 2)))
    blocks = out_words.reshape(N // 128, 128, K // 128, 16).transpose(0, 2, 1, 3)   # [T][B][r][i]
    return np.ascontiguousarray(blocks).reshape(-1).view(np.uint8)


@pytest.mark.parametrize("N,K", [(128, 128), (256, 640), (4096, 4096)])
def test_tile_w4_is_the_documented_permutation(N, K):
    rng = np.random.default_rng(N + K)
    packed = rng.integers(0, 256, size=(N, K // 2), dtype=np.uint8)
    pd = torch.from_numpy(packed).cuda()
    tiled = spear.spear_tile_w4(pd)
    torch.cuda.synchronize()
    got = tiled.cpu().numpy().reshape(-1)
    assert np.array_equal(got, _tile_order_numpy(packed, N, K))
    with pytest.raises(spear.SpearError):                 # K not a multiple of 128
        spear.spear_tile_w4(pd[:, : (K // 2) - 32].contiguous())


@pytest.mark.parametrize("M", [1, 8, 16, 32, 64])
def test_tiled_planner_runs(M):
    d = dev(1)
    L = d.L
    plan = spear.spear_gemm_plan_tiled(M, L.N, L.K, L.rank)
    assert plan.kernel_id == spear.SPEAR_KERNEL_STREAM_RK and plan.flags & spear.SPEAR_PLAN_W4_TILES
    ws = spear.alloc_workspace(plan.workspace_bytes)
    check_close(host_f64(d.run(M, plan, ws)), d.ref(M), True, f"tiled planner M={M}")
    ok_status(ws)


def test_w4eclayer_with_both_code_orders():
    # A layer holding both code orders plans each batch size on the order measured faster (the
    # tile order on decode-mlp at M = 1), passes the matching codes, and matches the oracle.
    d = dev(2)
    L = d.L
    lay = spear.W4ECLayer(d.packed, d.scale, d.zero, d.ec, tiled=d.tiled)
    for M in (1, 8):
        p = lay.plan(M)
        assert bool(p.flags & spear.SPEAR_PLAN_W4_TILES) == (p.kernel_id == spear.SPEAR_KERNEL_STREAM_RK)
        y = lay(d.x(M))
        torch.cuda.synchronize()
        rows = np.arange(M)
        check_close(host_f64(y)[rows], d.ref(M, rows=rows), True, f"W4ECLayer both orders M={M}")
        assert spear.spear_get_device_status(lay.workspace) == 0
    assert lay.plan(1).kernel_id == spear.SPEAR_KERNEL_STREAM_RK
