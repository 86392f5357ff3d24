"""The C-ABI library on the host: it loads, exports what include/spear.h declares, and
rejects bad arguments before launching anything (no GPU is needed for any of this)."""
import ctypes
import math
import os
import re
import subprocess

import pytest

import w4_gemm_error_channel_b200 as spear

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "spear.h")

OK, INVALID, SHAPE, MISALIGNED, WS_SMALL = 0, 1, 2, 3, 4


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"SPEAR_API\s+[\w\s\*]+?\b(spear_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for fn in ("spear_pack_w4", "spear_gemm_plan", "spear_w4ec_gemm", "spear_debug_unpack_w4",
               "spear_status_string", "spear_get_device_status", "spear_version"):
        assert fn in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(spear.LIB_PATH)
    for fn in declared_functions():
        assert hasattr(lib, fn), fn
    out = subprocess.run(["nm", "-D", "--defined-only", spear.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = {ln.split()[-1] for ln in out.splitlines() if " T " in ln}
    missing = [fn for fn in declared_functions() if fn not in exported]
    assert not missing, missing


def test_status_strings_and_version():
    for code in range(7):
        assert spear.spear_status_string(code)
    assert spear.spear_status_string(99) == "unknown status"
    assert spear.spear_version() >= 100


def _plan(M, N, K, r):
    p = spear.spear_plan()
    return spear._lib.spear_gemm_plan(M, N, K, r, -1, ctypes.byref(p)), p


@pytest.mark.parametrize("M,N,K,r", [(1, 4096, 4096, 64), (16, 4096, 4096, 64), (64, 22016, 4096, 64),
                                     (2048, 4096, 14336, 128), (4, 512, 512, 16), (4096, 16384, 2048, 0),
                                     (256, 2048, 8192, 32), (7, 128, 64, 0)])
def test_plan_is_consistent(M, N, K, r):
    st, p = _plan(M, N, K, r)
    assert st == OK
    assert p.kernel_id in (spear.SPEAR_KERNEL_SPLITK, spear.SPEAR_KERNEL_TC05)
    assert N % p.tile_n == 0
    k_slice = ((K + p.split_k - 1) // p.split_k + 63) // 64 * 64
    assert (p.split_k - 1) * k_slice < K          # no empty K slice
    assert p.workspace_bytes >= 128 * 1024
    if r:
        assert p.workspace_bytes >= 128 * 1024 + 4 * M * r


@pytest.mark.parametrize("M,N,K,r,want", [(1, 100, 4096, 0, SHAPE), (1, 4096, 100, 0, SHAPE),
                                          (1, 4096, 4096, 8, SHAPE), (1, 4096, 4096, 72, SHAPE),
                                          (1, 4096, 4096, 512, SHAPE), (-1, 4096, 4096, 0, INVALID),
                                          (1, 0, 4096, 0, INVALID), (70000, 4096, 4096, 0, SHAPE)])
def test_plan_rejects_bad_shapes(M, N, K, r, want):
    st, _ = _plan(M, N, K, r)
    assert st == want


def _gemm(M=4, N=512, K=512, x=0x1000, packed=0x2000, scale=0x3000, zero=0x4000, y=0x5000, ws=0x6000,
          ws_bytes=1 << 30, ec=None, y_dtype=0, plan=None):
    P = ctypes.c_void_p
    return spear._lib.spear_w4ec_gemm(plan, P(x), M, N, K, P(packed), P(scale), P(zero), ec, P(y), y_dtype, P(ws),
                                      ws_bytes, None)


def test_gemm_host_checks_return_before_launch():
    # Fake, never-dereferenced addresses: every case below must fail (or finish) on the host.
    assert _gemm(x=0) == INVALID
    assert _gemm(y=0) == INVALID
    assert _gemm(ws=0) == INVALID
    assert _gemm(y_dtype=7) == INVALID
    assert _gemm(N=500) == SHAPE
    assert _gemm(K=100) == SHAPE
    assert _gemm(x=0x1008) == MISALIGNED
    assert _gemm(packed=0x2001) == MISALIGNED
    assert _gemm(ws=0x6004) == MISALIGNED
    assert _gemm(ws_bytes=1024) == WS_SMALL
    assert _gemm(M=0) == OK               # empty batch: nothing to launch
    assert _gemm(M=0, x=0, y=0) == OK     # ... and may come without activation/output buffers
    ec = spear.spear_ec(0x7000, 0x8000, 0x9000, 0.0, 16)
    assert _gemm(ec=ctypes.byref(ec), ws_bytes=1024) == WS_SMALL
    bad = spear.spear_ec(0x7000, 0, 0x9000, 0.0, 16)
    assert _gemm(ec=ctypes.byref(bad)) == INVALID
    nan = spear.spear_ec(0x7000, 0x8000, 0x9000, math.nan, 16)
    assert _gemm(ec=ctypes.byref(nan)) == INVALID
    r8 = spear.spear_ec(0x7000, 0x8000, 0x9000, 0.0, 8)
    assert _gemm(ec=ctypes.byref(r8)) == SHAPE
    mis = spear.spear_ec(0x7008, 0x8000, 0x9000, 0.0, 16)
    assert _gemm(ec=ctypes.byref(mis)) == MISALIGNED


def test_gemm_rejects_bad_plans():
    st, p = _plan(4, 512, 512, 0)
    assert st == OK
    for field, val in (("kernel_id", 9), ("split_k", 0), ("split_k", 9), ("tile_n", 48), ("tile_m", 12)):
        q = spear.spear_plan.from_buffer_copy(p)
        setattr(q, field, val)
        assert _gemm(plan=ctypes.byref(q)) == INVALID, field
    # tcgen05 plans: 256 weight rows only with 128-token tiles; token widths 128, 160, 192, 256.
    # Plan flags: only SPEAR_PLAN_SEPARATE_EC (1).
    for kid, fl in ((1, 2), (1, 3), (2, 2), (2, 3)):
        q = spear.spear_plan.from_buffer_copy(p)
        q.kernel_id, q.flags = kid, fl
        if kid == 2:
            q.tile_n, q.split_k, q.tile_m = 128, 1, 128
        assert _gemm(plan=ctypes.byref(q)) == INVALID, (kid, fl)
    for tile_n, tile_m in ((256, 256), (256, 160), (64, 128), (128, 144)):
        q = spear.spear_plan.from_buffer_copy(p)
        q.kernel_id, q.split_k, q.tile_n, q.tile_m = 2, 1, tile_n, tile_m
        assert _gemm(plan=ctypes.byref(q)) == INVALID, (tile_n, tile_m)


def test_pack_and_unpack_host_checks():
    P = ctypes.c_void_p
    lib = spear._lib
    assert lib.spear_pack_w4(P(0), 1, 8, 8, P(0x2000), P(0x3000), P(0x4000), None) == INVALID
    assert lib.spear_pack_w4(P(0x1000), 5, 8, 8, P(0x2000), P(0x3000), P(0x4000), None) == INVALID
    assert lib.spear_pack_w4(P(0x1000), 1, 8, 7, P(0x2000), P(0x3000), P(0x4000), None) == SHAPE
    assert lib.spear_pack_w4(P(0x1000), 1, 0, 8, P(0x2000), P(0x3000), P(0x4000), None) == INVALID
    assert lib.spear_pack_w4(P(0x1004), 1, 8, 8, P(0x2000), P(0x3000), P(0x4000), None) == MISALIGNED
    assert lib.spear_debug_unpack_w4(P(0x1000), P(0x2000), 8, 8, P(0), P(0), None) == INVALID
    assert lib.spear_debug_unpack_w4(P(0x1000), P(0x2000), 8, 9, P(0x3000), P(0), None) == SHAPE
    assert lib.spear_get_device_status(P(0), 0, None) == INVALID


def test_prepared_layer_rejects_host_tensors():
    import torch
    with pytest.raises(ValueError):
        spear.W4ECLayer(torch.zeros((128, 32), dtype=torch.uint8), torch.zeros(128, dtype=torch.float16),
                        torch.zeros(128, dtype=torch.float16))


def test_mlp_gate_host_checks():
    # The optional bottleneck-MLP gate: all four arrays or none, 1 <= H <= 64, 16-byte aligned,
    # alpha not NaN; the no-allocation entry point takes the scalar gate only.  Fake, never
    # dereferenced addresses: every case is decided on the host.
    def ec(**kw):
        e = spear.spear_ec(0x7000, 0x8000, 0x9000, 0.0, 16)
        e.gate_w1, e.gate_b1, e.gate_w2, e.gate_b2, e.gate_hidden, e.alpha = 0xA000, 0xB000, 0xC000, 0xD000, 8, 1.0
        for k, v in kw.items():
            setattr(e, k, v)
        return e
    for kw, want in (({"gate_b1": 0}, INVALID), ({"gate_w2": 0}, INVALID), ({"gate_hidden": 0}, INVALID),
                     ({"gate_hidden": 65}, INVALID), ({"alpha": math.nan}, INVALID), ({"gate_w1": 0xA004}, MISALIGNED),
                     ({"gate_b2": 0xD008}, MISALIGNED)):
        e = ec(**kw)
        assert _gemm(ec=ctypes.byref(e)) == want, kw
    e = ec()
    P = ctypes.c_void_p
    assert spear._lib.spear_w4ec_gemm_noalloc(None, P(0x1000), 4, 512, 512, P(0x2000), P(0x3000), P(0x4000),
                                              ctypes.byref(e), P(0x5000), 0, None) == INVALID


def test_plan_update_and_semifused_workspace():
    # The semi-fused prefill plan (tcgen05 kernel + SPEAR_PLAN_SEPARATE_EC) keeps the fp32 main
    # term [M][N] in the workspace after u (bf16 [M][r], padded to 256 bytes).
    M, N, K, r = 300, 512, 512, 16
    st, p = _plan(M, N, K, r)
    assert st == OK
    q = spear.spear_plan.from_buffer_copy(p)
    q.kernel_id, q.tile_n, q.split_k, q.tile_m, q.flags = 2, 128, 1, 128, 0
    assert spear._lib.spear_plan_update(ctypes.byref(q), M, N, K, r) == OK
    fused = q.workspace_bytes
    assert fused == (128 + 1024) * 1024 + (M * r * 2 + 255) // 256 * 256
    q.flags = spear.SPEAR_PLAN_SEPARATE_EC
    assert spear._lib.spear_plan_update(ctypes.byref(q), M, N, K, r) == OK
    assert q.workspace_bytes == fused + M * N * 4
    ec = spear.spear_ec(0x7000, 0x8000, 0x9000, 0.0, r)
    assert _gemm(M=M, N=N, K=K, ec=ctypes.byref(ec), plan=ctypes.byref(q), ws_bytes=q.workspace_bytes - 1) == WS_SMALL
    # Without a compensator the flag changes nothing.
    assert spear._lib.spear_plan_update(ctypes.byref(q), M, N, K, 0) == OK
    assert q.workspace_bytes == (128 + 1024) * 1024
    # Bad fields and shapes are refused and leave the plan as it was.
    before = bytes(q)
    q2 = spear.spear_plan.from_buffer_copy(q)
    q2.flags = 2
    assert spear._lib.spear_plan_update(ctypes.byref(q2), M, N, K, r) == INVALID
    assert spear._lib.spear_plan_update(ctypes.byref(q), M, 500, K, r) == SHAPE
    assert spear._lib.spear_plan_update(None, M, N, K, r) == INVALID
    assert bytes(q) == before
    with pytest.raises(spear.SpearError):
        spear.spear_plan_update(q2, M, N, K, r)


def _measured_rows():
    inc = os.path.join(os.path.dirname(spear.__file__), "csrc", "plan_table.inc")
    rows = []
    for line in open(inc):
        if line.startswith("{"):
            v = line.strip().strip("{},").split(",")
            rows.append(tuple(int(t) for t in v[:9]))
    return rows


def test_planner_returns_every_measured_plan():
    # The dispatcher hands out, at each measured shape, the plan the table recorded for it (row-order
    # codes), and every row -- tile-order rows included -- is a plan spear_plan_update accepts.
    rows = _measured_rows()
    assert len(rows) > 50
    for (M, N, K, e, kern, tile_n, split, tile_m, flags) in rows:
        r = 32 if e else 0
        q = spear.spear_plan()
        q.kernel_id, q.tile_n, q.split_k, q.tile_m, q.flags = kern, tile_n, split, tile_m, flags
        if kern == spear.SPEAR_KERNEL_SPLITK:
            q.tile_m = 8 if M <= 8 else (16 if M <= 16 else 32)
        assert spear._lib.spear_plan_update(ctypes.byref(q), M, N, K, r) == OK, (M, N, K, e, kern, split)
        if kern == spear.SPEAR_KERNEL_STREAM_RK:
            continue
        st, p = _plan(M, N, K, r)
        assert st == OK
        assert (p.kernel_id, p.split_k) == (kern, split), (M, N, K, e)
        if kern == spear.SPEAR_KERNEL_SPLITK:
            assert p.tile_n == tile_n
        else:
            assert p.tile_m == tile_m


def test_tc05_k_split_plan_checks():
    # The tcgen05 kernel's K split: 2, 4 or 8 CTAs per tile (a cluster), 128 weight rows, token
    # tiles of 128 or 256, (K / 64) divisible by the split, fused compensator only.
    M, N, K, r = 256, 2048, 8192, 32
    st, p = _plan(M, N, K, r)
    assert st == OK

    def upd(split, tile_m=128, tile_n=128, flags=0, k=K, rank=r):
        q = spear.spear_plan.from_buffer_copy(p)
        q.kernel_id, q.tile_n, q.split_k, q.tile_m, q.flags = 2, tile_n, split, tile_m, flags
        return spear._lib.spear_plan_update(ctypes.byref(q), M, N, k, rank), q
    for split in (1, 2, 4, 8):
        for tile_m in (128, 256):
            st, q = upd(split, tile_m)
            assert st == OK, (split, tile_m)
            assert q.workspace_bytes == upd(1, tile_m)[1].workspace_bytes   # no workspace of its own
    for kw in ({"split": 3}, {"split": 16}, {"split": 0}, {"split": 2, "tile_n": 256},
               {"split": 4, "tile_m": 160}, {"split": 8, "tile_m": 192},
               {"split": 8, "k": 64 * 12}, {"split": 2, "flags": spear.SPEAR_PLAN_SEPARATE_EC}):
        assert upd(**kw)[0] == INVALID, kw
    # Each owner's share of the token tile is a multiple of 16: 160 tokens split 2 ways (80 each),
    # 192 split 2 or 4 ways (96, 48).
    assert upd(2, tile_m=160)[0] == OK
    assert upd(4, tile_m=192)[0] == OK
    # The split does not combine with the separate-EC flag, with or without a compensator.
    assert upd(2, flags=spear.SPEAR_PLAN_SEPARATE_EC, rank=0)[0] == INVALID


def test_grouped_host_checks():
    # Group-wise scales: groups of a multiple of 128 dividing K for the layer (any even divisor for
    # the packer), compensator rank <= 128.  Fake, never-dereferenced addresses throughout.
    P, lib = ctypes.c_void_p, spear._lib
    pack = lambda W=0x1000, N=256, K=512, G=128, packed=0x2000, dt=1: lib.spear_pack_w4_grouped(
        P(W), dt, N, K, G, P(packed), P(0x3000), P(0x4000), None)
    assert pack(W=0) == INVALID
    assert pack(G=0) == INVALID
    assert pack(G=7) == SHAPE
    assert pack(G=96) == SHAPE            # does not divide 512
    assert pack(packed=0x2008) == MISALIGNED
    out = ctypes.c_size_t()
    ws = lambda M=300, N=512, K=512, G=128, r=0: lib.spear_grouped_workspace_bytes(M, N, K, G, r, ctypes.byref(out))
    assert ws() == OK and out.value == (128 + 1024) * 1024
    assert ws(r=16) == OK and out.value == (128 + 1024) * 1024 + (300 * 16 * 2 + 255) // 256 * 256 + 300 * 512 * 4
    for kw, want in (({"G": 64}, SHAPE), ({"G": 384}, SHAPE), ({"r": 144}, SHAPE), ({"r": 8}, SHAPE),
                     ({"N": 500}, SHAPE), ({"M": -1}, INVALID)):
        assert ws(**kw) == want, kw
    assert lib.spear_grouped_workspace_bytes(1, 512, 512, 128, 0, None) == INVALID

    def gemm(M=4, N=512, K=512, G=128, x=0x1000, y=0x5000, wsp=0x6000, ws_bytes=1 << 30, ec=None):
        return lib.spear_w4ec_gemm_grouped(P(x), M, N, K, G, P(0x2000), P(0x3000), P(0x4000), ec, P(y), 0, P(wsp),
                                           ws_bytes, None)
    assert gemm(x=0) == INVALID
    assert gemm(wsp=0) == INVALID
    assert gemm(G=64) == SHAPE
    assert gemm(x=0x1008) == MISALIGNED
    assert gemm(ws_bytes=1024) == WS_SMALL
    assert gemm(M=0) == OK
    big = spear.spear_ec(0x7000, 0x8000, 0x9000, 0.0, 144)
    assert gemm(ec=ctypes.byref(big)) == SHAPE
    e16 = spear.spear_ec(0x7000, 0x8000, 0x9000, 0.0, 16)
    assert gemm(ec=ctypes.byref(e16), ws_bytes=(128 + 1024) * 1024) == WS_SMALL


def test_plan_update_decode_plans():
    # Split-K decode plans: the separate EC pass keeps the fp32 main term of one launch (at most
    # 256 tokens) after the zeroed part; tile and split rules are those of spear_w4ec_gemm.
    M, N, K, r = 16, 4096, 4096, 64
    st, p = _plan(M, N, K, r)
    assert st == OK
    q = spear.spear_plan.from_buffer_copy(p)
    q.kernel_id, q.tile_n, q.split_k, q.tile_m, q.flags = 1, 32, 4, 16, 0
    assert spear._lib.spear_plan_update(ctypes.byref(q), M, N, K, r) == OK
    fused = q.workspace_bytes
    assert fused == (128 + 1024) * 1024
    q.flags = spear.SPEAR_PLAN_SEPARATE_EC
    assert spear._lib.spear_plan_update(ctypes.byref(q), M, N, K, r) == OK
    assert q.workspace_bytes == fused + M * N * 4
    assert spear._lib.spear_plan_update(ctypes.byref(q), 1000, N, K, r) == OK
    assert q.workspace_bytes == fused + 256 * N * 4
    for field, val in (("split_k", 3), ("tile_n", 24), ("tile_m", 12), ("flags", 4)):
        bad = spear.spear_plan.from_buffer_copy(q)
        setattr(bad, field, val)
        assert spear._lib.spear_plan_update(ctypes.byref(bad), M, N, K, r) == INVALID, field
    # tcgen05: 256 weight rows need 128-token tiles and N % 256 == 0; rank at most 128.
    t = spear.spear_plan.from_buffer_copy(q)
    t.kernel_id, t.tile_n, t.split_k, t.tile_m, t.flags = 2, 256, 1, 128, 0
    assert spear._lib.spear_plan_update(ctypes.byref(t), 2048, N, K, r) == OK
    assert spear._lib.spear_plan_update(ctypes.byref(t), 2048, 4224, K, r) == INVALID
    t.tile_m = 256
    assert spear._lib.spear_plan_update(ctypes.byref(t), 2048, N, K, r) == INVALID
    t.tile_n, t.tile_m = 128, 256
    assert spear._lib.spear_plan_update(ctypes.byref(t), 2048, N, K, 144) == INVALID


def test_tiled_plan_and_tile_order_argument_checks():
    # Plans for codes in the tile order: the register-path stream kernel, flagged as such.
    p = spear.spear_plan()
    for M in (1, 8, 16, 32, 64):
        assert spear._lib.spear_gemm_plan_tiled(M, 4096, 4096, 64, -1, ctypes.byref(p)) == OK
        assert p.kernel_id == spear.SPEAR_KERNEL_STREAM_RK and p.flags & spear.SPEAR_PLAN_W4_TILES
        assert p.tile_m >= M and 4096 % p.split_k == 0
    for M, N, K, r in ((65, 4096, 4096, 64), (1, 4160, 4096, 64), (1, 4096, 4032, 64), (1, 4096, 4096, 144)):
        assert spear._lib.spear_gemm_plan_tiled(M, N, K, r, -1, ctypes.byref(p)) == SHAPE, (M, N, K, r)
    # Without the flag the register path is refused; the row-order kernels refuse the flag.
    assert spear._lib.spear_gemm_plan_tiled(4, 4096, 4096, 64, -1, ctypes.byref(p)) == OK
    q = spear.spear_plan.from_buffer_copy(p)
    q.flags &= ~spear.SPEAR_PLAN_W4_TILES
    assert spear._lib.spear_plan_update(ctypes.byref(q), 4, 4096, 4096, 64) == INVALID
    st, rows = _plan(4, 4096, 4096, 64)
    assert st == OK and not rows.flags & spear.SPEAR_PLAN_W4_TILES
    assert rows.kernel_id != spear.SPEAR_KERNEL_STREAM_RK           # row-order planning never picks it
    rows.flags |= spear.SPEAR_PLAN_W4_TILES
    assert spear._lib.spear_plan_update(ctypes.byref(rows), 4, 4096, 4096, 64) == INVALID
    # spear_tile_w4 checks its arguments before touching the device.
    tile = spear._lib.spear_tile_w4
    assert tile(None, 128, 128, ctypes.c_void_p(4096), None) == INVALID
    assert tile(ctypes.c_void_p(4096), 100, 128, ctypes.c_void_p(1 << 20), None) == SHAPE
    assert tile(ctypes.c_void_p(4096), 128, 192, ctypes.c_void_p(1 << 20), None) == SHAPE
    assert tile(ctypes.c_void_p(4104), 128, 128, ctypes.c_void_p(1 << 20), None) == MISALIGNED
    assert tile(ctypes.c_void_p(4096), 128, 128, ctypes.c_void_p(4096 + 16), None) == INVALID   # overlap


def test_plan_formats_picks_among_code_orders():
    p = spear.spear_plan()
    f = spear._lib.spear_gemm_plan_formats
    assert f(4, 4096, 4096, 64, -1, 0, ctypes.byref(p)) == INVALID
    assert f(4, 4096, 4096, 64, -1, 8, ctypes.byref(p)) == INVALID
    st, rows = _plan(4, 4096, 4096, 64)
    assert f(4, 4096, 4096, 64, -1, spear.SPEAR_W4_ROWS, ctypes.byref(p)) == OK
    assert (p.kernel_id, p.tile_n, p.split_k, p.tile_m, p.flags) == (rows.kernel_id, rows.tile_n, rows.split_k,
                                                                     rows.tile_m, rows.flags)
    assert f(4, 4096, 4096, 64, -1, spear.SPEAR_W4_TILES, ctypes.byref(p)) == OK
    assert p.kernel_id == spear.SPEAR_KERNEL_STREAM_RK and p.flags & spear.SPEAR_PLAN_W4_TILES
    for M, N, K in ((1, 22016, 4096), (16, 4096, 4096), (64, 22016, 4096), (2048, 4096, 14336)):
        assert f(M, N, K, 64, -1, spear.SPEAR_W4_ROWS | spear.SPEAR_W4_TILES, ctypes.byref(p)) == OK
        # The plan's flag names the order it reads; only the register path reads tiles.
        assert bool(p.flags & spear.SPEAR_PLAN_W4_TILES) == (p.kernel_id == spear.SPEAR_KERNEL_STREAM_RK)
        assert spear._lib.spear_plan_update(ctypes.byref(p), M, N, K, 64) == OK
