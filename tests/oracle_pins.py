"""Pins for the CPU oracle: checks against facts fixed outside the oracle itself.

Each ``pin_*`` function takes an ``oracle.Oracle`` and raises AssertionError when
the oracle disagrees with something the pages or the mathematics fix:

* library routines: numpy's IEEE binary16 rounding, numpy float64 matmul/exp;
* exact arithmetic: ``fractions.Fraction`` brute force on 8x8 problems;
* closed forms: weights already on the int4 grid round-trip exactly; power-of-two
  row scaling; gate limits (b_g = -inf gives g = 0 exactly, +inf gives g = 1);
  rank-0 / zero factors reduce to the plain W4 layer;
* hand-derived rows in tests/golden/rtn_hand_rows.txt.

The same functions run against deliberately broken builds of the oracle in
test_oracle_mutants.py, which shows each plausible mistake fails at least one pin.
"""
from __future__ import annotations

import math
import os
from fractions import Fraction

import numpy as np

from synthetic import bf16_bits_from_f32, f32_from_bf16_bits

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


# ----------------------------------------------------------------------------- helpers

def f16_bits_to_f64(bits) -> np.ndarray:
    return np.asarray(bits, np.uint16).view(np.float16).astype(np.float64)


def numpy_unpack(packed: np.ndarray, K: int) -> np.ndarray:
    """Documented nibble layout: byte b holds k=2b in bits 0..3, k=2b+1 in bits 4..7."""
    q = np.empty((packed.shape[0], K), np.uint8)
    q[:, 0::2] = packed & 0xF
    q[:, 1::2] = packed >> 4
    return q


def small_layer(seed: int, M: int, N: int, K: int, r: int, b_g: float = 0.3):
    rng = np.random.default_rng(seed)
    x = bf16_bits_from_f32(rng.standard_normal((M, K)).astype(np.float32))
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    A = bf16_bits_from_f32((rng.standard_normal((K, r)) * 0.05).astype(np.float32))
    B = bf16_bits_from_f32((rng.standard_normal((r, N)) * 0.05).astype(np.float32))
    wg = bf16_bits_from_f32((rng.standard_normal(K) * 0.1).astype(np.float32))
    return x, W, A, B, wg, b_g


def read_golden_rows():
    rows = []
    cur = {}
    with open(os.path.join(GOLDEN, "rtn_hand_rows.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *vals = line.split()
            if key == "w":
                cur = {"w": [float(v) for v in vals]}
            elif key == "q":
                cur["q"] = [int(v) for v in vals]
            elif key in ("s", "z"):
                cur[key] = int(vals[0], 16)
                if key == "z":
                    rows.append(cur)
    return rows


# ----------------------------------------------------------------------------- number formats

def pin_f16_encoder(o):
    """The oracle's binary16 encoder equals numpy's IEEE round-to-nearest-even cast."""
    rng = np.random.default_rng(11)
    vals = [rng.standard_normal(400) * sc for sc in (1e-7, 3e-6, 1e-4, 0.02, 1.0, 300.0, 3e4)]
    # exact midpoints between neighbouring binary16 values (ties), subnormal and normal
    h = rng.integers(0, 0x7BFE, 600).astype(np.uint16)
    a = h.view(np.float16).astype(np.float64)
    b = (h + 1).astype(np.uint16).view(np.float16).astype(np.float64)
    vals.append((a + b) / 2)
    vals.append(np.array([0.0, -0.0, 65504.0, 65519.0, 65520.0, 1e9, 2.0 ** -25, 2.0 ** -24, 6.0e-5]))
    v = np.concatenate(vals).astype(np.float32)
    v = np.concatenate([v, -v])
    with np.errstate(over="ignore"):
        want = v.astype(np.float16).view(np.uint16)
    got = np.array([o.f32_to_f16_bits(float(x)) for x in v], np.uint16)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, f"binary16 encoder mismatch at {v[bad[:5]]}: {got[bad[:5]]} vs {want[bad[:5]]}"
    dec = np.array([o.f16_bits_to_f64(int(x)) for x in want[:200]])
    assert np.array_equal(dec, want[:200].view(np.float16).astype(np.float64))


# ----------------------------------------------------------------------------- quantiser

def pin_golden_rows(o):
    """Hand-derived rows (tests/golden/rtn_hand_rows.txt) quantise as derived."""
    rows = read_golden_rows()
    W = np.array([r["w"] for r in rows], np.float32)
    q, s, z = o.quantize_rtn(W)
    for i, r in enumerate(rows):
        assert list(q[i]) == r["q"], f"row {i}: q {list(q[i])} != {r['q']}"
        assert int(s[i]) == r["s"], f"row {i}: s {hex(s[i])} != {hex(r['s'])}"
        assert int(z[i]) == r["z"], f"row {i}: z {hex(z[i])} != {hex(r['z'])}"


def pin_grid_round_trip(o):
    """Weights already on the int4 grid, W = (q - z) s, come back bit-exactly."""
    rng = np.random.default_rng(12)
    N, K = 96, 128
    q = rng.integers(0, 16, (N, K)).astype(np.uint8)
    for n in range(N):  # every row holds both ends of the code range
        i, j = rng.choice(K, 2, replace=False)
        q[n, i], q[n, j] = 0, 15
    z = rng.integers(0, 16, N)
    z[:4] = [0, 15, 8, 1]
    e = rng.integers(-12, 0, N)
    m = rng.integers(0, 1024, N)
    s = (1024 + m) * np.exp2(e - 10.0)
    W = ((q.astype(np.float64) - z[:, None]) * s[:, None]).astype(np.float32)
    assert np.array_equal(W.astype(np.float64), (q.astype(np.float64) - z[:, None]) * s[:, None])
    q2, s2, z2 = o.quantize_rtn(W)
    assert np.array_equal(q2, q), "codes not recovered"
    assert np.array_equal(f16_bits_to_f64(s2), s), "scales not recovered"
    assert np.array_equal(f16_bits_to_f64(z2), z.astype(np.float64)), "zeros not recovered"
    packed = o.pack_nibbles(q)
    assert np.array_equal(packed, (q[:, 0::2] | (q[:, 1::2] << 4)).astype(np.uint8)), "nibble layout"
    assert np.array_equal(o.unpack_nibbles(packed, K), q)
    p2, s3, z3 = o.pack_w4(W)
    assert np.array_equal(p2, packed) and np.array_equal(s3, s2) and np.array_equal(z3, z2)


def _argmin_tie_even(cands, dist, parity_of):
    best = min(dist)
    idx = [i for i, d in enumerate(dist) if d == best]
    if len(idx) == 1:
        return cands[idx[0]], False
    even = [i for i in idx if parity_of(cands[i]) % 2 == 0]
    return cands[even[0]], True


def pin_rtn_bruteforce(o):
    """Each code is the nearest grid point in exact arithmetic (ties to an even q - z)."""
    rng = np.random.default_rng(13)
    W = (rng.standard_normal((8, 8)) * 0.02).astype(np.float32)
    W[5] = np.abs(W[5])            # all-positive row: lo = 0
    W[6] = -np.abs(W[6])           # all-negative row: hi = 0
    W[7] *= 37.0                   # another binade
    q, s_bits, z_bits = o.quantize_rtn(W)
    s_val = f16_bits_to_f64(s_bits)
    z_val = f16_bits_to_f64(z_bits)
    near = 0
    for n in range(8):
        row = [Fraction(float(v)) for v in W[n]]
        lo, hi = min(min(row), Fraction(0)), max(max(row), Fraction(0))
        want_s = np.float16(float((hi - lo) / 15))  # one rounding of the exact quotient
        assert s_val[n] == float(want_s), f"row {n}: scale {s_val[n]} != {float(want_s)}"
        S = Fraction(s_val[n])
        zc = list(range(16))
        zbest, _ = _argmin_tie_even(zc, [abs(-lo - zz * S) for zz in zc], lambda v: v)
        assert z_val[n] == zbest, f"row {n}: zero {z_val[n]} != {zbest}"
        for k in range(8):
            d = [abs(row[k] - (qq - zbest) * S) for qq in range(16)]
            srt = sorted(d)
            if srt[1] - srt[0] < S * Fraction(1, 10 ** 6) and srt[1] != srt[0]:
                near += 1
                continue
            qbest, _ = _argmin_tie_even(list(range(16)), d, lambda v: v - zbest)
            assert q[n, k] == qbest, f"({n},{k}): code {q[n, k]} != {qbest}"
    assert near <= 2


def pin_scale_pow2(o):
    """Scaling a row by 2^j leaves q and z unchanged and scales s by exactly 2^j."""
    rng = np.random.default_rng(14)
    W = (rng.standard_normal((16, 64)) * 0.02).astype(np.float32)
    q, s, z = o.quantize_rtn(W)
    for j in (-3, -1, 1, 4):
        q2, s2, z2 = o.quantize_rtn((W * np.float32(2.0 ** j)).astype(np.float32))
        assert np.array_equal(q2, q) and np.array_equal(z2, z)
        assert np.array_equal(f16_bits_to_f64(s2), f16_bits_to_f64(s) * 2.0 ** j)


# ----------------------------------------------------------------------------- layer

def _independent_What(packed, s_bits, z_bits, K):
    q = numpy_unpack(packed, K).astype(np.float64)
    return (q - f16_bits_to_f64(z_bits)[:, None]) * f16_bits_to_f64(s_bits)[:, None]


def pin_main_term_vs_numpy(o):
    """Plain W4 layer == numpy float64 matmul of x and the dequantised weights."""
    x, W, A, B, wg, b_g = small_layer(21, M=7, N=48, K=96, r=8)
    packed, s, z = o.pack_w4(W)
    What = _independent_What(packed, s, z, 96)
    assert np.array_equal(o.dequant_w4(packed, s, z, 96), What)
    y = o.w4ec_gemm(x, packed, s, z)
    want = f32_from_bf16_bits(x).astype(np.float64) @ What.T
    assert np.allclose(y, want, rtol=0, atol=1e-12 * np.abs(want).max())


def pin_ec_vs_numpy(o):
    """t = x A, p = x w_g + b_g, g = 1/(1+e^-p) and the EC term, against numpy fp64."""
    x, W, A, B, wg, b_g = small_layer(22, M=6, N=32, K=64, r=16, b_g=-0.7)
    xf = f32_from_bf16_bits(x).astype(np.float64)
    Af = f32_from_bf16_bits(A).astype(np.float64)
    Bf = f32_from_bf16_bits(B).astype(np.float64)
    wf = f32_from_bf16_bits(wg).astype(np.float64)
    t, p, g = o.ec_gate(x, A, wg, b_g)
    assert np.allclose(t, xf @ Af, rtol=0, atol=1e-13 * np.abs(t).max())
    p_want = xf @ wf + np.float64(np.float32(b_g))
    assert np.allclose(p, p_want, rtol=0, atol=1e-13 * np.abs(p_want).max())
    assert np.allclose(g, 1.0 / (1.0 + np.exp(-p_want)), rtol=1e-14, atol=0)
    packed, s, z = o.pack_w4(W)
    y = o.w4ec_gemm(x, packed, s, z, A, B, wg, b_g)
    y0 = o.w4ec_gemm(x, packed, s, z)
    ec = g[:, None] * ((xf @ Af) @ Bf)
    assert np.allclose(y - y0, ec, rtol=0, atol=1e-12 * np.abs(y).max())


def pin_gate_limits(o):
    """b_g=-inf -> g=0 (plain layer, exactly); b_g=+inf -> g=1; rank 0 / A=0 / B=0 -> plain."""
    x, W, A, B, wg, _ = small_layer(23, M=5, N=32, K=64, r=8)
    packed, s, z = o.pack_w4(W)
    y0 = o.w4ec_gemm(x, packed, s, z)
    assert np.array_equal(o.w4ec_gemm(x, packed, s, z, A, B, wg, float("-inf")), y0)
    zA = np.zeros_like(A)
    zB = np.zeros_like(B)
    assert np.array_equal(o.w4ec_gemm(x, packed, s, z, zA, B, wg, 0.5), y0)
    assert np.array_equal(o.w4ec_gemm(x, packed, s, z, A, zB, wg, 0.5), y0)
    assert np.array_equal(o.w4ec_gemm(x, packed, s, z, A[:, :0], B[:0], wg, 0.5), y0)
    xf = f32_from_bf16_bits(x).astype(np.float64)
    full = y0 + (xf @ f32_from_bf16_bits(A).astype(np.float64)) @ f32_from_bf16_bits(B).astype(np.float64)
    y1 = o.w4ec_gemm(x, packed, s, z, A, B, wg, float("inf"))
    assert np.allclose(y1, full, rtol=0, atol=1e-12 * np.abs(full).max())
    _, p, g = o.ec_gate(x, A, wg, 0.0)
    _, pn, gn = o.ec_gate(x, A, (wg ^ 0x8000).astype(np.uint16), 0.0)  # w_g -> -w_g
    assert np.array_equal(pn, -p) and np.allclose(g + gn, 1.0, rtol=0, atol=1e-15)


def pin_bruteforce_rational(o):
    """8x8 layer in exact rationals (sigmoid of the exact pre-activation taken in fp64)."""
    M = N = K = 8
    r = 4
    x, W, A, B, wg, b_g = small_layer(24, M, N, K, r, b_g=0.25)
    packed, s, z = o.pack_w4(W)
    q = numpy_unpack(packed, K)
    S = [Fraction(float(v)) for v in f16_bits_to_f64(s)]
    Z = [Fraction(float(v)) for v in f16_bits_to_f64(z)]
    X = [[Fraction(float(v)) for v in row] for row in f32_from_bf16_bits(x)]
    Af = [[Fraction(float(v)) for v in row] for row in f32_from_bf16_bits(A)]
    Bf = [[Fraction(float(v)) for v in row] for row in f32_from_bf16_bits(B)]
    G = [Fraction(float(v)) for v in f32_from_bf16_bits(wg)]
    y = o.w4ec_gemm(x, packed, s, z, A, B, wg, b_g)
    for m in range(M):
        t = [sum(X[m][k] * Af[k][j] for k in range(K)) for j in range(r)]
        p = sum(X[m][k] * G[k] for k in range(K)) + Fraction(float(np.float32(b_g)))
        g = Fraction(1.0 / (1.0 + math.exp(-float(p))))
        for n in range(N):
            main = sum(X[m][k] * (int(q[n, k]) - Z[n]) * S[n] for k in range(K))
            ec = sum(t[j] * Bf[j][n] for j in range(r))
            want = float(main + g * ec)
            assert abs(y[m, n] - want) <= 1e-13 * max(1.0, abs(want)), (m, n, y[m, n], want)


def pin_sampled_and_prefix(o):
    """Sampled evaluation equals the full product; token rows are independent."""
    x, W, A, B, wg, b_g = small_layer(25, M=9, N=64, K=128, r=16)
    packed, s, z = o.pack_w4(W)
    y = o.w4ec_gemm(x, packed, s, z, A, B, wg, b_g)
    rng = np.random.default_rng(5)
    mi = rng.integers(0, 9, 50)
    ni = rng.integers(0, 64, 50)
    ys = o.w4ec_gemm_sampled(x, packed, s, z, A, B, wg, b_g, mi, ni)
    assert np.array_equal(ys, y[mi, ni])
    assert np.array_equal(o.w4ec_gemm(x[:4], packed, s, z, A, B, wg, b_g), y[:4])


def pin_mlp_gate(o):
    """Bottleneck-MLP gate (gamma(t) = sigmoid(W2 relu(W1 t + b1) + b2), u = alpha gamma t) against
    cases that reduce to the scalar-gate oracle or to the plain layer, plus its invariances."""
    x, W, A, B, wg, _ = small_layer(31, M=5, N=32, K=64, r=8)
    packed, s, z = o.pack_w4(W)
    r, H = 8, 3
    rng = np.random.default_rng(32)
    W1 = rng.standard_normal((H, r)).astype(np.float32)
    b1 = rng.standard_normal(H).astype(np.float32) * 0.1
    W2 = rng.standard_normal((r, H)).astype(np.float32)
    b2 = rng.standard_normal(r).astype(np.float32) * 0.1
    y0 = o.w4ec_gemm(x, packed, s, z)
    zeros_wg = np.zeros_like(wg)
    scale = 1e-12 * np.abs(y0).max()
    # gamma = 1 (W2 = 0, b2 = +inf): the scalar gate at g = 1.
    inf = np.full(r, np.inf, np.float32)
    y1 = o.w4ec_gemm_mlp(x, packed, s, z, A, B, W1, b1, np.zeros_like(W2), inf, 1.0)
    assert np.allclose(y1, o.w4ec_gemm(x, packed, s, z, A, B, zeros_wg, float("inf")), rtol=0, atol=scale)
    # gamma = 0 (b2 = -inf): the plain layer.
    assert np.allclose(o.w4ec_gemm_mlp(x, packed, s, z, A, B, W1, b1, np.zeros_like(W2), -inf, 1.0), y0,
                       rtol=0, atol=scale)
    # Dead hidden units (b1 very negative) and equal output biases c: gamma = sigmoid(c) everywhere,
    # the scalar gate with w_g = 0, b_g = c.
    c = np.float32(-0.75)
    yd = o.w4ec_gemm_mlp(x, packed, s, z, A, B, W1, np.full(H, -1e30, np.float32), W2, np.full(r, c, np.float32), 1.0)
    assert np.allclose(yd, o.w4ec_gemm(x, packed, s, z, A, B, zeros_wg, float(c)), rtol=0, atol=scale)
    # One hidden unit that reads rank j0 (W1 = e_j0, a large b1 keeps relu linear, b2 = -b1):
    # gamma_j = sigmoid(t_j0) for every j, the scalar gate with w_g = column j0 of A.
    j0 = 5
    e = np.zeros((1, r), np.float32)
    e[0, j0] = 1.0
    big = np.float32(100.0)
    ys = o.w4ec_gemm_mlp(x, packed, s, z, A, B, e, np.array([big], np.float32), np.ones((r, 1), np.float32),
                         np.full(r, -big, np.float32), 1.0)
    col = np.ascontiguousarray(A[:, j0])
    assert np.allclose(ys, o.w4ec_gemm(x, packed, s, z, A, B, col, 0.0), rtol=0, atol=1e-9 * np.abs(ys).max())
    # alpha scales the compensator term linearly.
    ya = o.w4ec_gemm_mlp(x, packed, s, z, A, B, W1, b1, W2, b2, 1.0)
    yb = o.w4ec_gemm_mlp(x, packed, s, z, A, B, W1, b1, W2, b2, 2.5)
    assert np.allclose(yb - y0, 2.5 * (ya - y0), rtol=0, atol=scale)
    assert np.abs(ya - y0).max() > 1e3 * scale
    # Duplicated hidden units with halved output weights leave the layer unchanged.
    yu = o.w4ec_gemm_mlp(x, packed, s, z, A, B, np.vstack([W1, W1]), np.concatenate([b1, b1]),
                         np.hstack([W2, W2]) / 2, b2, 1.0)
    assert np.allclose(yu, ya, rtol=0, atol=scale)


def pin_grouped(o):
    """Group-wise scales (G consecutive k per scale and zero-point): G = K is the per-channel
    layer; for G < K the layer equals numpy's matmul with weights dequantised group by group
    (scales broadcast with np.repeat), plus the EC term; each group's RTN error stays within
    half its step, and no group's step exceeds its row's per-channel step."""
    x, W, A, B, wg, b_g = small_layer(41, M=5, N=24, K=256, r=8)
    K, N = 256, 24
    packed, s, z = o.pack_w4(W)
    pg, sg, zg = o.pack_w4_grouped(W, K)
    assert np.array_equal(pg, packed) and np.array_equal(sg[:, 0], s) and np.array_equal(zg[:, 0], z)
    y_pc = o.w4ec_gemm(x, packed, s, z, A, B, wg, b_g)
    y_g = o.w4ec_gemm_grouped(x, pg, sg, zg, K, A, B, wg, b_g)
    assert np.allclose(y_g, y_pc, rtol=0, atol=1e-12 * np.abs(y_pc).max())
    xf = f32_from_bf16_bits(x).astype(np.float64)
    t, _, g = o.ec_gate(x, A, wg, b_g)
    ec = g[:, None] * (t @ f32_from_bf16_bits(B).astype(np.float64))
    for G in (32, 64, 128):
        pg, sg, zg = o.pack_w4_grouped(W, G)
        assert pg.shape == (N, K // 2) and sg.shape == (N, K // G)
        q = numpy_unpack(pg, K).astype(np.float64)
        sf = np.repeat(f16_bits_to_f64(sg), G, axis=1)
        zf = np.repeat(f16_bits_to_f64(zg), G, axis=1)
        What = (q - zf) * sf
        assert np.all(np.abs(W.astype(np.float64) - What) <= 0.5 * sf * (1 + 1e-6) + 1e-12)
        assert np.all(f16_bits_to_f64(sg) <= f16_bits_to_f64(s)[:, None])
        want = xf @ What.T
        y = o.w4ec_gemm_grouped(x, pg, sg, zg, G)
        assert np.allclose(y, want, rtol=0, atol=1e-12 * np.abs(want).max())
        y = o.w4ec_gemm_grouped(x, pg, sg, zg, G, A, B, wg, b_g)
        assert np.allclose(y, want + ec, rtol=0, atol=1e-12 * np.abs(want + ec).max())
    # A change inside one group moves only that group's codes, scale and zero-point.
    G = 64
    W2 = W.copy()
    W2[3, 70] = 0.5
    pa, sa, za = o.pack_w4_grouped(W, G)
    pb, sb, zb = o.pack_w4_grouped(W2, G)
    diff_s = np.argwhere(sa != sb)
    assert diff_s.tolist() == [[3, 1]] and (za != zb).sum() <= 1
    qa, qb = numpy_unpack(pa, K), numpy_unpack(pb, K)
    rows, cols = np.nonzero(qa != qb)
    assert set(rows.tolist()) == {3} and cols.min() >= 64 and cols.max() < 128


ALL_PINS = [pin_f16_encoder, pin_golden_rows, pin_grid_round_trip, pin_rtn_bruteforce, pin_scale_pow2,
            pin_main_term_vs_numpy, pin_ec_vs_numpy, pin_gate_limits, pin_bruteforce_rational,
            pin_sampled_and_prefix, pin_mlp_gate, pin_grouped]
