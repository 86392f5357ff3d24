"""The semi-fused prefill path (tcgen05 kernel with SPEAR_PLAN_SEPARATE_EC) against the oracle,
through the C ABI: the EC tiles alone on the library's side stream, the main tiles alone on the
caller's stream, joined by the up-projection kernel (y = fp32 main term + u B).

Besides parity: the path leaves the workspace's control words zeroed, so fused and semi-fused
calls can share a workspace in any order; and a CUDA graph captured from the caller's stream holds
the two tcgen05 launches as parallel branches that the up-projection joins."""
import os
import re

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

ZEROED = (128 + 1024) * 1024


def _plan(M, N, K, r, tile_m=128, wrows=128, semi=True):
    p = spear.spear_gemm_plan(M, N, K, r)
    p.kernel_id, p.tile_n, p.split_k, p.tile_m = spear.SPEAR_KERNEL_TC05, wrows, 1, tile_m
    p.flags = spear.SPEAR_PLAN_SEPARATE_EC if semi else 0
    return spear.spear_plan_update(p, M, N, K, r)


def _layer_dev(L):
    packed, scale, zero = spear.spear_pack_w4(to_dev(L.W))
    ec = spear.EC(to_dev_bf16(L.A_bits), to_dev_bf16(L.B_bits), to_dev_bf16(L.wg_bits), L.b_g)
    return packed, scale, zero, ec


def _ref(L, M, rows=None):
    p, s, z = oracle.pack_w4(L.W)
    xs = L.x(M) if rows is None else L.x(M)[rows]
    return oracle.w4ec_gemm(xs, p, s, z, L.A_bits, L.B_bits, L.wg_bits, L.b_g)


def _run(L, M, plan, y_dtype=torch.bfloat16, ws=None):
    packed, scale, zero, ec = _layer_dev(L)
    ws = spear.alloc_workspace(plan.workspace_bytes) if ws is None else ws
    y = spear.spear_w4ec_gemm(to_dev_bf16(L.x(M)), packed, scale, zero, ec, y_dtype=y_dtype, plan=plan,
                              workspace=ws)
    torch.cuda.synchronize()
    assert spear.spear_get_device_status(ws) == 0
    return y, ws


@pytest.mark.parametrize("tile_m,wrows", [(128, 128), (256, 128), (160, 128), (128, 256)])
@pytest.mark.parametrize("r", [16, 64, 128])
@pytest.mark.parametrize("M", [1, 128, 300])
def test_semifused_small(M, r, tile_m, wrows):
    L = make_layer("semi", 101 + r + M, M, 512, 512, r, outlier_frac=0.02, outlier_scale=10.0, b_g=0.3)
    y, ws = _run(L, M, _plan(M, L.N, L.K, r, tile_m, wrows))
    check_close(host_f64(y), _ref(L, M), True, f"semi-fused M={M} r={r} tile_m={tile_m} rows={wrows}")
    assert int(ws[:ZEROED].count_nonzero().item()) == 0


def test_semifused_fp32_and_gate_off():
    L = make_layer("semi", 121, 200, 384, 640, 64, b_g=-1.0)
    y, _ = _run(L, 200, _plan(200, L.N, L.K, 64), y_dtype=torch.float32)
    check_close(host_f64(y), _ref(L, 200), False, "semi-fused fp32")
    # b_g = -inf: g = 0, u = 0, so the result equals the plain layer from the same kernel bit for bit.
    packed, scale, zero, ec = _layer_dev(L)
    ec.b_g = float("-inf")
    x = to_dev_bf16(L.x(200))
    p = _plan(200, L.N, L.K, 64)
    y_off = spear.spear_w4ec_gemm(x, packed, scale, zero, ec, plan=p, workspace=spear.alloc_workspace(p.workspace_bytes))
    y_plain = spear.spear_w4ec_gemm(x, packed, scale, zero, None, plan=_plan(200, L.N, L.K, 0, semi=False))
    assert torch.equal(y_off, y_plain)


@pytest.mark.parametrize("M,r,H", [(128, 64, 16), (300, 128, 64)])
def test_semifused_mlp_gate(M, r, H):
    L = make_layer("semim", 130 + M + r, M, 256, 512, r, outlier_frac=0.01, outlier_scale=20.0, ec_std=0.05)
    rng = np.random.default_rng(H)
    W1 = (rng.standard_normal((H, r)) * 0.5).astype(np.float32)
    b1 = (rng.standard_normal(H) * 0.2).astype(np.float32)
    W2 = (rng.standard_normal((r, H)) * 0.5).astype(np.float32)
    b2 = (rng.standard_normal(r) * 0.5).astype(np.float32)
    packed, scale, zero = spear.spear_pack_w4(to_dev(L.W))
    ec = spear.EC(to_dev_bf16(L.A_bits), to_dev_bf16(L.B_bits), to_dev_bf16(L.wg_bits), L.b_g,
                  gate_w1=to_dev(W1), gate_b1=to_dev(b1), gate_w2=to_dev(W2), gate_b2=to_dev(b2), alpha=1.3)
    plan = _plan(M, L.N, L.K, r, 256)
    ws = spear.alloc_workspace(plan.workspace_bytes)
    y = spear.spear_w4ec_gemm(to_dev_bf16(L.x(M)), packed, scale, zero, ec, plan=plan, workspace=ws)
    torch.cuda.synchronize()
    assert spear.spear_get_device_status(ws) == 0
    p, s, z = oracle.pack_w4(L.W)
    ref = oracle.w4ec_gemm_mlp(L.x(M), p, s, z, L.A_bits, L.B_bits, W1, b1, W2, b2, 1.3)
    check_close(host_f64(y), ref, True, f"semi-fused MLP gate M={M} r={r} H={H}")


@pytest.mark.parametrize("tile_m", [128, 256])
def test_semifused_prefill_sampled(tile_m):
    # The prefill layer (M=2048, N=4096, K=14336, r=128), sampled rows against the oracle, and the
    # whole output against the fused path (the two differ only in the last fp32 sum's rounding).
    L = config_layers(3)[0]
    M = 2048
    rows = np.array([0, 1, 255, 256, 1031, 2047])
    y, ws = _run(L, M, _plan(M, L.N, L.K, L.rank, tile_m))
    check_close(host_f64(y)[rows], _ref(L, M, rows), True, f"semi-fused prefill tile_m={tile_m}")
    y_fused, _ = _run(L, M, _plan(M, L.N, L.K, L.rank, tile_m, semi=False))
    d = (y.float() - y_fused.float()).abs()
    rms = float(y_fused.float().pow(2).mean().sqrt())
    assert float(d.max()) <= 1e-2 * rms + float(y_fused.float().abs().max()) * 2.0 ** -7


def test_semifused_and_fused_share_a_workspace():
    L = make_layer("semis", 141, 300, 512, 512, 64, b_g=0.2)
    M = 300
    semi = _plan(M, L.N, L.K, 64)
    ws = spear.alloc_workspace(semi.workspace_bytes)
    ref = _ref(L, M)
    for p in (_plan(M, L.N, L.K, 64, semi=False), semi, _plan(M, L.N, L.K, 64, 256, semi=False), semi):
        y, _ = _run(L, M, p, ws=ws)
        check_close(host_f64(y), ref, True, f"shared workspace flags={p.flags}")
        assert int(ws[:ZEROED].count_nonzero().item()) == 0


def _dot_structure(text):
    """Kernel nodes (id -> label text) and edges of a graph dumped as DOT."""
    decl = list(re.finditer(r'"?(graph_\d+_node_\d+)"?\s*\[', text))
    nodes = {}
    for i, m in enumerate(decl):             # an id may also open an edge's attribute list
        end = decl[i + 1].start() if i + 1 < len(decl) else len(text)
        nodes[m.group(1)] = nodes.get(m.group(1), "") + text[m.end():end]
    edges = re.findall(r'"?(graph_\d+_node_\d+)"?\s*->\s*"?(graph_\d+_node_\d+)"?', text)
    return nodes, edges


def _reaches(edges, a, b):
    seen, todo = set(), [a]
    while todo:
        n = todo.pop()
        if n == b:
            return True
        if n in seen:
            continue
        seen.add(n)
        todo.extend(d for s, d in edges if s == n)
    return False


def test_semifused_graph_is_a_dag_with_parallel_branches(tmp_path):
    L = make_layer("semig", 151, 300, 512, 512, 32, b_g=0.1)
    M = 300
    packed, scale, zero, ec = _layer_dev(L)
    plan = _plan(M, L.N, L.K, 32)
    ws = spear.alloc_workspace(plan.workspace_bytes)
    x = to_dev_bf16(L.x(M))
    y = torch.empty((M, L.N), dtype=torch.bfloat16, device="cuda")
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):                       # warm-up outside the capture
        spear.spear_w4ec_gemm(x, packed, scale, zero, ec, y=y, plan=plan, workspace=ws)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    y.zero_()
    g = torch.cuda.CUDAGraph(keep_graph=True)        # keeps the captured graph for the DOT dump
    g.enable_debug_mode()
    with torch.cuda.graph(g):
        spear.spear_w4ec_gemm(x, packed, scale, zero, ec, y=y, plan=plan, workspace=ws)
    dot = os.path.join(str(tmp_path), "semifused.dot")
    g.debug_dump(dot)
    g.instantiate()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    assert spear.spear_get_device_status(ws) == 0
    check_close(host_f64(y), _ref(L, M), True, "semi-fused graph replay")
    assert int(ws[:ZEROED].count_nonzero().item()) == 0

    text = open(dot).read()
    nodes, edges = _dot_structure(text)
    tc = [n for n, lab in nodes.items() if "tc05" in lab]
    up = [n for n, lab in nodes.items() if "ec_up_add" in lab]
    assert len(tc) == 2 and len(up) == 1, (sorted(nodes), tc, up, text[:3000])
    a, b = tc
    assert not _reaches(edges, a, b) and not _reaches(edges, b, a), "the two tcgen05 launches are serialised"
    assert _reaches(edges, a, up[0]) and _reaches(edges, b, up[0])
    g.reset()
