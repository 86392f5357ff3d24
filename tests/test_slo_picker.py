"""The SLO-constrained prefill chunk picker (host only, no GPU): closed forms on hand-made latency
tables, the bisection against a brute-force scan, monotonicity, the effect of where compensators
sit, and argument errors."""
import math
import os

import pytest

import w4_gemm_error_channel_b200 as spear
from synthetic.workloads import SWEEP_EC_LAYERS, SWEEP_LAYERS, SWEEP_LINEARS, SWEEP_RANK

OK, INVALID, SHAPE = 0, 1, 2

# One linear whose call takes 10 + 0.5 M us, measured at M = 1 and M = 1001.
LINE = [(1, 256, 512, 0, 10.5), (1001, 256, 512, 0, 510.5)]
ONE = [(256, 512, 0, 1)]


def model(ec_layers=SWEEP_EC_LAYERS):
    """The 16-layer model of config 4 as (N, K, rank, count)."""
    n_ec = len(ec_layers)
    return ([(N, K, SWEEP_RANK, n_ec) for (_, N, K) in SWEEP_LINEARS] +
            [(N, K, 0, SWEEP_LAYERS - n_ec) for (_, N, K) in SWEEP_LINEARS])


def test_interpolation_closed_forms():
    for M, want in ((0, 0.0), (1, 10.5), (101, 60.5), (500, 260.0), (1001, 510.5), (2002, 1021.0)):
        assert math.isclose(spear.spear_predict_step_us(ONE, M, lut=LINE), want, rel_tol=1e-12), M
    assert math.isclose(spear.spear_predict_step_us([(256, 512, 0, 3)], 101, fixed_us=7.0, lut=LINE), 7 + 3 * 60.5)


def test_pick_closed_form():
    # 16 decode tokens, granule 16, target 200 us: 10 + 0.5 (16 + C) <= 200  ->  C <= 364  ->  352.
    chunk, pred = spear.spear_pick_prefill_chunk(ONE, 16, 4096, 200.0, granule=16, lut=LINE)
    assert (chunk, pred) == (352, 194.0)
    # max_chunk caps it; a fixed time shifts it: 30 + 10 + 0.5 (16 + C) <= 200 -> C <= 304.
    assert spear.spear_pick_prefill_chunk(ONE, 16, 100, 200.0, granule=16, lut=LINE)[0] == 96
    assert spear.spear_pick_prefill_chunk(ONE, 16, 4096, 200.0, granule=16, fixed_us=30.0, lut=LINE)[0] == 304
    # Target below the decode-only step: chunk 0, predicted above the target.
    chunk, pred = spear.spear_pick_prefill_chunk(ONE, 16, 4096, 5.0, granule=16, lut=LINE)
    assert chunk == 0 and pred == 18.0


def test_samples_are_made_monotone():
    lut = [(100, 256, 512, 0, 50.0), (200, 256, 512, 0, 40.0), (300, 256, 512, 0, 60.0)]
    assert spear.spear_predict_step_us(ONE, 200, lut=lut) == 50.0
    assert spear.spear_predict_step_us(ONE, 150, lut=lut) == 50.0
    assert spear.spear_predict_step_us(ONE, 250, lut=lut) == 55.0
    # Duplicate rows of one M: the larger time.
    assert spear.spear_predict_step_us(ONE, 100, lut=lut + [(100, 256, 512, 0, 52.0)]) == 52.0


def test_builtin_table_reads_back_and_is_monotone():
    table = spear.spear_latency_table()
    assert len(table) > 10 and all(M >= 1 and us > 0 for (M, _, _, _, us) in table)
    # One row per shape: the fastest of the dispatcher's rows for it (both code orders).
    keys = [(M, N, K, e) for (M, N, K, e, _) in table]
    assert len(keys) == len(set(keys))
    inc = os.path.join(os.path.dirname(spear.__file__), "csrc", "plan_table.inc")
    fastest = {}
    for line in open(inc):
        if line.startswith("{"):
            v = [float(t) for t in line.strip().strip("{},").split(",")]
            k = tuple(int(t) for t in v[:4])
            fastest[k] = min(fastest.get(k, math.inf), v[9])
    assert {k: round(us, 3) for (*k, us) in map(tuple, table) for k in [tuple(k)]} == \
        {k: round(us, 3) for k, us in fastest.items()}
    lin = model()
    prev = 0.0
    for M in range(0, 4097, 16):
        t = spear.spear_predict_step_us(lin, M)
        assert t >= prev
        prev = t
    # At a measured M the step is the sum of the measured calls, each raised to the largest time
    # measured for its shape at a smaller batch (the predictor makes every shape's samples
    # nondecreasing in M).
    row = {(M, N, K, e): us for (M, N, K, e, us) in table}

    def envelope(M, N, K, e):
        return max(us for (m, n, k, ee), us in row.items() if (n, k, ee) == (N, K, e) and m <= M)
    for M in (1, 16, 256, 4096):
        want = sum(c * envelope(M, N, K, int(r > 0)) for (N, K, r, c) in lin)
        assert math.isclose(spear.spear_predict_step_us(lin, M), want, rel_tol=1e-12)


@pytest.mark.parametrize("slo", [300.0, 1000.0, 2000.0, 5000.0, 9000.0, 20000.0])
@pytest.mark.parametrize("granule", [64, 128])
def test_bisection_matches_brute_force(slo, granule):
    lin, D, cap = model(), 16, 4096 - 16
    chunk, pred = spear.spear_pick_prefill_chunk(lin, D, cap, slo, granule=granule)
    ok = [c * granule for c in range(cap // granule + 1) if spear.spear_predict_step_us(lin, D + c * granule) <= slo]
    assert chunk == (max(ok) if ok else 0)
    assert chunk % granule == 0 and chunk <= cap
    assert math.isclose(pred, spear.spear_predict_step_us(lin, D + chunk), rel_tol=1e-12)


def test_more_compensators_never_allow_a_larger_chunk():
    dense = (0, 1, 2, 3, 4, 5, 6, 7, 8, 9, 10, 11, 12, 13, 14, 15)
    for slo in (1500.0, 3000.0, 6000.0):
        c0 = spear.spear_pick_prefill_chunk(model(()), 16, 4080, slo)[0]
        c4 = spear.spear_pick_prefill_chunk(model(), 16, 4080, slo)[0]
        c16 = spear.spear_pick_prefill_chunk(model(dense), 16, 4080, slo)[0]
        assert c0 >= c4 >= c16, (slo, c0, c4, c16)
    assert spear.spear_predict_step_us(model(dense), 1040) > spear.spear_predict_step_us(model(()), 1040)


def test_errors():
    lib, P = spear._lib, None
    chunk, pred = spear.ctypes.c_int64(), spear.ctypes.c_double()
    la = spear._linears(ONE)
    lp, ln = spear._lut(LINE)
    call = lambda **kw: lib.spear_pick_prefill_chunk(
        kw.get("la", la), kw.get("n", 1), kw.get("D", 16), kw.get("cap", 4096), kw.get("g", 16), kw.get("slo", 200.0),
        kw.get("fixed", 0.0), kw.get("lp", lp), kw.get("ln", ln), spear.ctypes.byref(chunk), spear.ctypes.byref(pred))
    assert call() == OK and chunk.value == 352
    for kw in ({"n": 0}, {"D": -1}, {"cap": -1}, {"g": 0}, {"slo": 0.0}, {"slo": math.nan}, {"fixed": -1.0},
               {"ln": 0}, {"la": P}):
        assert call(**kw) == INVALID, kw
    bad = spear._lut([(0, 256, 512, 0, 1.0)])
    assert call(lp=bad[0], ln=1) == INVALID
    # A linear with no row of its shape: unsupported, unless it runs zero times.
    assert call(la=spear._linears([(384, 512, 0, 1)])) == SHAPE
    assert call(la=spear._linears([(256, 512, 0, 1), (384, 512, 0, 0)]), n=2) == OK
    assert call(la=spear._linears([(256, 512, 16, 1)])) == SHAPE     # the table has this shape without EC only
    with pytest.raises(spear.SpearError):
        spear.spear_predict_step_us([(256, 512, 0, 1)], 70000, lut=LINE)
    # decode tokens + chunk never exceed 65536 tokens.
    c, _ = spear.spear_pick_prefill_chunk(ONE, 65500, 4096, 1e9, granule=16, lut=LINE)
    assert c == 32


# ----------------------------------------------------------------------------- properties
from hypothesis import given, settings, strategies as st  # noqa: E402


def _py_T(samples, M):
    """The documented reading of a latency table, restated: nondecreasing samples (larger time for
    a repeated M, then the running maximum), linear interpolation, flat below, proportional above."""
    if M <= 0:
        return 0.0
    by_m = {}
    for m, us in samples:
        by_m[m] = max(by_m.get(m, 0.0), us)
    pts = sorted(by_m.items())
    run, mono = 0.0, []
    for m, us in pts:
        run = max(run, us)
        mono.append((m, run))
    if M <= mono[0][0]:
        return mono[0][1]
    if M >= mono[-1][0]:
        return mono[-1][1] * M / mono[-1][0]
    for (m0, t0), (m1, t1) in zip(mono, mono[1:]):
        if m0 <= M <= m1:
            return t0 + (t1 - t0) * (M - m0) / (m1 - m0)


_sample = st.tuples(st.integers(1, 8192), st.floats(0.5, 5000.0, allow_nan=False))
_shape = st.tuples(st.sampled_from([(256, 512), (1024, 256), (2048, 2048)]), st.booleans(),
                   st.lists(_sample, min_size=1, max_size=6), st.integers(0, 5))


@settings(max_examples=80, deadline=None)
@given(shapes=st.lists(_shape, min_size=1, max_size=4, unique_by=lambda s: (s[0], s[1])),
       D=st.integers(0, 512), cap=st.integers(0, 9000), granule=st.sampled_from([1, 16, 64, 128, 1000]),
       slo=st.floats(1.0, 1e5, allow_nan=False), fixed=st.floats(0.0, 500.0, allow_nan=False))
def test_picker_properties(shapes, D, cap, granule, slo, fixed):
    lut, lin = [], []
    for (N, K), has_ec, samples, count in shapes:
        lut += [(m, N, K, int(has_ec), us) for (m, us) in samples]
        lin.append((N, K, 16 if has_ec else 0, count))
    step = lambda M: fixed + sum(c * _py_T([(m, us) for (m, n, k, e, us) in lut if (n, k, e) == (N, K, int(r > 0))], M)
                                 for (N, K, r, c) in lin)
    for M in (0, 1, D, D + 7, 4096, 65536):
        got = spear.spear_predict_step_us(lin, M, fixed_us=fixed, lut=lut)
        assert math.isclose(got, step(M), rel_tol=1e-9, abs_tol=1e-9), M
    chunk, pred = spear.spear_pick_prefill_chunk(lin, D, cap, slo, granule=granule, fixed_us=fixed, lut=lut)
    room = min(cap, 65536 - D)
    assert chunk % granule == 0 and 0 <= chunk <= room
    assert math.isclose(pred, step(D + chunk), rel_tol=1e-9, abs_tol=1e-9)
    if step(D) <= slo:
        assert pred <= slo
        if chunk + granule <= room:
            assert step(D + chunk + granule) > slo
    else:
        assert chunk == 0
    a, b = sorted((D, D + chunk + 3))
    assert spear.spear_predict_step_us(lin, a, fixed_us=fixed, lut=lut) <= \
        spear.spear_predict_step_us(lin, b, fixed_us=fixed, lut=lut) + 1e-9
