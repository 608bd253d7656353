"""Pins for the oracle: each test checks the oracle against something other
than itself -- brute force over tiny code tables and tiny routings, closed
forms, library conversions (torch's float8 / bfloat16 casts), exact error
bounds, and the routing table printed on "[feat] A5 deep fused moe
supported" (Testing).  CPU only."""
import itertools
import os

import numpy as np
import pytest
import torch

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
RNG = np.random.default_rng(12345)


# ---------------------------------------------------------------------------
# small-float encoders: brute force over the code tables written from the
# OCP format definitions (independent of the oracle's rounding arithmetic)
# ---------------------------------------------------------------------------

def _e4m3_table():
    vals = []
    for c in range(0x7F):  # 0x7F is NaN
        e, m = c >> 3, c & 7
        vals.append(m * 2.0 ** -9 if e == 0 else (1 + m / 8) * 2.0 ** (e - 7))
    return np.array(vals)


def _e2m1_table():
    return np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def _brute_encode(x, table, sign_bit):
    """Nearest table value, ties to the even code, beyond the top -> top."""
    x = np.asarray(x, np.float64)
    a = np.abs(x)
    hi = np.clip(np.searchsorted(table, a), 1, len(table) - 1)
    lo = hi - 1
    dlo, dhi = a - table[lo], table[hi] - a
    pick = np.where(dlo < dhi, lo, np.where(dhi < dlo, hi, np.where(lo % 2 == 0, lo, hi)))
    pick = np.where(a >= table[-1], len(table) - 1, pick)
    return (pick | np.where(np.signbit(x), sign_bit, 0)).astype(np.uint8)


def _all_bf16_finite_f32():
    b = np.arange(1 << 16, dtype=np.uint32) << 16
    f = b.view(np.float32)
    return f[np.isfinite(f)]


def _midpoint_probe(table):
    """Every midpoint between neighbouring codes, and its fp32 neighbours."""
    mids = ((table[1:] + table[:-1]) / 2).astype(np.float32)
    mids = np.concatenate([mids, np.float32([table[-1] * 1.0625, table[-1] * 1.5, 1e30])])
    out = [mids]
    for d in (1, 2):
        out.append(np.nextafter(mids, np.float32(np.inf)))
        out.append(np.nextafter(mids, np.float32(0)))
        mids = out[-2]
    v = np.concatenate(out)
    return np.concatenate([v, -v])


def _random_f32(n, lo_exp, hi_exp):
    mag = 2.0 ** RNG.uniform(lo_exp, hi_exp, n)
    sign = np.where(RNG.random(n) < 0.5, -1.0, 1.0)
    return (mag * sign).astype(np.float32)


@pytest.mark.parametrize("probe", ["bf16", "midpoints", "random"])
def test_e4m3_encoder_matches_brute_force(probe):
    table = _e4m3_table()
    x = {"bf16": _all_bf16_finite_f32, "midpoints": lambda: _midpoint_probe(table),
         "random": lambda: _random_f32(2_000_000, -14, 10)}[probe]()
    got = oracle.e4m3_encode(x)
    want = _brute_encode(x, table, 0x80)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, (x[bad[:5]], got[bad[:5]], want[bad[:5]])


def test_e4m3_encoder_matches_torch_float8_in_range():
    # torch's float8_e4m3fn cast rounds to nearest even but does not saturate:
    # compare where no saturation is involved (|x| < 464 rounds to <= 448).
    x = np.concatenate([_all_bf16_finite_f32(), _random_f32(1_000_000, -12, 8.85)])
    x = x[np.abs(x) < 464]
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = oracle.e4m3_encode(x)
    assert np.array_equal(got, ref)


def test_e4m3_nan_and_saturation():
    got = oracle.e4m3_encode(np.float32([np.nan, 448, 449, 1e38, -1e38, np.inf, -np.inf, 0.0, -0.0]))
    assert list(got) == [0x7F, 0x7E, 0x7E, 0x7E, 0xFE, 0x7E, 0xFE, 0x00, 0x80]


@pytest.mark.parametrize("probe", ["bf16", "midpoints", "random"])
def test_e2m1_encoder_matches_brute_force(probe):
    table = _e2m1_table()
    x = {"bf16": _all_bf16_finite_f32, "midpoints": lambda: _midpoint_probe(table),
         "random": lambda: _random_f32(2_000_000, -4, 4)}[probe]()
    got = oracle.e2m1_encode(x)
    want = _brute_encode(x, table, 0x8)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, (x[bad[:5]], got[bad[:5]], want[bad[:5]])


def test_decoders_invert_encoders_on_every_code():
    for c in range(256):
        if c & 0x7F == 0x7F:
            continue
        v = oracle.e4m3_decode(np.uint8([c]))[0]
        assert oracle.e4m3_encode(np.float32([v]))[0] == c
    for c in range(16):
        v = oracle.e2m1_decode(np.uint8([c]))[0]
        assert oracle.e2m1_encode(np.float32([v]))[0] == c


def test_decoders_give_nan_for_the_e4m3_nan_codes():
    dec = oracle.e4m3_decode(np.uint8([0x7F, 0xFF, 0x7E, 0xFE]))
    assert np.isnan(dec[0]) and np.isnan(dec[1]) and list(dec[2:]) == [448.0, -448.0]
    # and the combine of a row holding one turns that element into NaN only
    d = np.zeros(32, np.uint8)
    d[[0, 5]] = [0x7F, 0x38]                       # NaN, 1.0
    y = oracle.dequant_row("mxfp8", d, np.uint8([127]), 32)
    assert np.isnan(y[0]) and y[5] == 1.0 and np.all(y[[1, 2, 3, 4]] == 0)


def test_bf16_rounding_matches_torch():
    x = np.concatenate([_random_f32(1_000_000, -130, 127),
                        # exact ties: low half 0x8000 with even and odd kept bit
                        (np.arange(0, 1 << 16, 7, dtype=np.uint32) << 16 | 0x8000).view(np.float32)])
    x = x[np.isfinite(x)]
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(oracle.f32_to_bf16(x), ref)


# ---------------------------------------------------------------------------
# e8m0 exponent: closed form 2^(X-1) < amax/qmax <= 2^X (exact in float64)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("qmax", [448.0, 6.0])
def test_mx_exponent_is_ceil_log2(qmax):
    amax = np.concatenate([
        _random_f32(500_000, -140, 127), _all_bf16_finite_f32(),
        (2.0 ** np.arange(-149, 120) * qmax).astype(np.float32)])
    amax = np.abs(amax[np.isfinite(amax) & (amax != 0)]).astype(np.float32)
    X = oracle.mx_exponent(amax, qmax).astype(np.int64)
    v = (amax / np.float32(qmax)).astype(np.float64)  # the IEEE fp32 division, widened exactly
    inside = (X > -127) & (X < 127) & (v > 0)
    Xi = X[inside]
    assert np.all(v[inside] <= np.ldexp(1.0, Xi))
    assert np.all(v[inside] > np.ldexp(1.0, Xi - 1))
    low = ~inside & (X == -127)
    assert np.all((v[low] <= 2.0 ** -127))
    assert oracle.mx_exponent(np.float32([0.0]), qmax)[0] == 0


# ---------------------------------------------------------------------------
# row quantisation: exact error bounds and the codes that must appear
# ---------------------------------------------------------------------------

def _bf16_row(n, scale=1.0, seed=0):
    r = np.random.default_rng(seed)
    return synth.to_bf16_bits((r.standard_normal(n) * scale).astype(np.float32))


def _f(bits):
    return oracle.bf16_to_f32(bits).astype(np.float64)


def test_quant_bf16_is_a_copy():
    x = _bf16_row(1024)
    d, s = oracle.quant_row("bf16", x)
    assert s.size == 0 and np.array_equal(d.view(np.uint16), x)


@pytest.mark.parametrize("seed", range(6))
def test_quant_int8_token_bounds(seed):
    H = 4096
    x = _bf16_row(H, scale=10.0 ** (seed - 3), seed=seed)
    if seed == 5:  # outlier channels, as in the skewed workload
        f = oracle.bf16_to_f32(x).copy()
        f[::97] *= 50
        x = synth.to_bf16_bits(f)
    d, s = oracle.quant_row("int8_token", x)
    q = d.view(np.int8).astype(np.float64)
    sinv = float(s.view(np.float32)[0])
    xf = _f(x)
    amax = np.abs(xf).max()
    assert sinv == pytest.approx(amax / 127, rel=2 ** -23)
    assert np.abs(q).max() == 127 and np.all(np.abs(q) <= 127)
    # q = rint(fl(x * fl(127/amax))): within half a step plus two fp32 roundings
    err = np.abs(xf - q * sinv)
    assert np.all(err <= 0.5 * sinv * (1 + 2 ** -20) + np.abs(xf) * 2 ** -21)
    # the element of largest magnitude maps to +-127 with its sign
    i = int(np.argmax(np.abs(xf)))
    assert q[i] == np.sign(xf[i]) * 127


def _e4m3_elem_bound(v):
    """|v - e4m3(v)| for |v| <= 448: half a code step (2^-4 relative in the
    normal range, 2^-10 absolute among subnormals)."""
    return np.maximum(np.abs(v) * 2.0 ** -4, 2.0 ** -10)


@pytest.mark.parametrize("qmax", [448.0, 127.0])
@pytest.mark.parametrize("seed", range(4))
def test_quant_e4m3_b128_bounds(qmax, seed):
    H = 7168
    x = _bf16_row(H, scale=10.0 ** (seed - 2), seed=seed)
    d, s = oracle.quant_row("e4m3_b128", x, e4m3_qmax=qmax)
    sinv = s.view(np.float32).astype(np.float64)
    dec = oracle.e4m3_decode(d).astype(np.float64).reshape(-1, 128)
    xf = _f(x).reshape(-1, 128)
    amax = np.abs(xf).max(axis=1)
    assert np.allclose(sinv, amax / qmax, rtol=2 ** -23, atol=0)
    v = xf * (qmax / amax)[:, None]          # the scaled values, exact in float64
    assert np.all(np.abs(v - dec) <= _e4m3_elem_bound(v) * (1 + 2 ** -18) + np.abs(v) * 2 ** -22)
    top = oracle.e4m3_encode(np.float32([qmax]))[0]
    assert np.all(np.abs(d.reshape(-1, 128).view(np.int8) & 0x7F).max(axis=1) == top)


@pytest.mark.parametrize("mode,qmax", [("mxfp8", 448.0), ("mxfp4", 6.0)])
@pytest.mark.parametrize("seed", range(4))
def test_quant_mx_bounds(mode, qmax, seed):
    H = 7168
    r = np.random.default_rng(seed)
    f = (r.standard_t(3, H) * 0.5 * 10.0 ** (seed - 1)).astype(np.float32)
    x = synth.to_bf16_bits(f)
    d, s = oracle.quant_row(mode, x)
    X = s.astype(np.int64) - 127
    assert np.all((s != 255))
    xf = _f(x).reshape(-1, 32)
    amax = np.abs(xf).max(axis=1)
    # ceil rule: amax * 2^-X lies in (qmax/2, qmax]
    scaled_amax = amax * np.ldexp(1.0, -X)
    assert np.all(scaled_amax <= qmax) and np.all(scaled_amax > qmax / 2)
    if mode == "mxfp8":
        dec = oracle.e4m3_decode(d).astype(np.float64).reshape(-1, 32)
        v = xf * np.ldexp(1.0, -X)[:, None]
        assert np.all(np.abs(v - dec) <= _e4m3_elem_bound(v))
    else:
        codes = np.stack([d & 0xF, d >> 4], axis=1).reshape(-1)  # element 2i = low nibble
        dec = oracle.e2m1_decode(codes).astype(np.float64).reshape(-1, 32)
        v = xf * np.ldexp(1.0, -X)[:, None]
        step = np.where(np.abs(v) < 2, 0.5, np.where(np.abs(v) < 4, 1.0, 2.0))
        assert np.all(np.abs(v - dec) <= step / 2)


def test_mxfp4_block_worked_by_hand():
    # A block whose amax is 6 has X = ceil(log2(6/6)) = 0, so the codes are the
    # e2m1 grid itself: 0,.5,1,1.5,2,3,4,6 -> codes 0..7, negatives add 8.
    vals = [0, 0.5, 1, 1.5, 2, 3, 4, 6, -0.5, -1, -1.5, -2, -3, -4, -6, 0] * 2
    x = synth.to_bf16_bits(np.float32(vals))
    d, s = oracle.quant_row("mxfp4", x)
    assert list(s) == [127]
    codes = [0, 1, 2, 3, 4, 5, 6, 7, 9, 10, 11, 12, 13, 14, 15, 0] * 2
    want = [codes[2 * i] | (codes[2 * i + 1] << 4) for i in range(16)]
    assert list(d) == want
    # doubling every value doubles the scale (X = 1) and keeps the codes
    d2, s2 = oracle.quant_row("mxfp4", synth.to_bf16_bits(np.float32(vals) * 2))
    assert list(s2) == [128] and np.array_equal(d2, d)


def test_mxfp8_block_worked_by_hand():
    # amax 448 -> X = 0: codes are the e4m3 encodings of the values themselves;
    # amax 1 -> X = ceil(log2(1/448)) = -8, every value is scaled by 256.
    vals = np.float32([448, -448, 1, -1, 0.5, 2 ** -9, 0, 3] + [0] * 24)
    d, s = oracle.quant_row("mxfp8", synth.to_bf16_bits(vals))
    assert list(s) == [127]
    assert list(d[:8]) == [0x7E, 0xFE, 0x38, 0xB8, 0x30, 0x01, 0x00, 0x44]
    d, s = oracle.quant_row("mxfp8", synth.to_bf16_bits(np.float32([1, -0.25] + [0] * 30)))
    assert list(s) == [127 - 8]
    assert list(d[:2]) == list(oracle.e4m3_encode(np.float32([256, -64])))


def test_zero_rows_use_unit_scale():
    x = np.zeros(256, np.uint16)
    d, s = oracle.quant_row("int8_token", x)
    assert not d.any() and s.view(np.float32)[0] == 1.0
    d, s = oracle.quant_row("e4m3_b128", x)
    assert not d.any() and np.all(s.view(np.float32) == 1.0)
    for m in ("mxfp8", "mxfp4"):
        d, s = oracle.quant_row(m, x)
        assert not d.any() and np.all(s == 127)


# ---------------------------------------------------------------------------
# layout: brute force over every routing of tiny shapes, closed forms
# ---------------------------------------------------------------------------

def _layout_by_definition(R, T, K, E, M, idx, align):
    """Counts straight from the definitions, one question per output."""
    N, L = R * T, E // R
    flat = [(n, k, int(idx[n][k])) for n in range(N) for k in range(K)]
    valid = lambda e: 0 <= e < E
    slot = np.full((N, K), -1, np.int64)
    for i, (n, k, e) in enumerate(flat):
        if valid(e):
            slot[n, k] = sum(1 for (_, _, e2) in flat[:i] if e2 == e)
    recv = np.array([sum(1 for (_, _, e2) in flat if e2 == e) for e in range(E)], dtype=np.int64)
    itr = np.array([[int(any(valid(e) and e // L == d for e in idx[n])) for d in range(R)]
                    for n in range(N)], dtype=np.int64).reshape(N, R)
    tpe = np.array([[sum(1 for t in range(T) for e in idx[r * T + t] if e == x) for x in range(E)]
                    for r in range(R)], dtype=np.int64).reshape(R, E)
    tpr = np.array([[itr[r * T:(r + 1) * T, d].sum() for d in range(R)] for r in range(R)])
    rounded = (recv + align - 1) // align * align
    eo = np.concatenate([[0], np.cumsum(rounded)])
    return slot, recv, itr, tpe, tpr, eo


def _check_layout(R, T, K, E, M, idx, align=1):
    idx = np.asarray(idx, np.int64).reshape(R * T, K)
    got = oracle.layout(R, T, K, E, M, idx, layout="packed", align=align)
    slot, recv, itr, tpe, tpr, eo = _layout_by_definition(R, T, K, E, M, idx, align)
    assert np.array_equal(got["token_slot"], slot)
    assert np.array_equal(got["recv_count"], recv)
    assert np.array_equal(got["is_token_in_rank"], itr)
    assert np.array_equal(got["tokens_per_expert"], tpe)
    assert np.array_equal(got["tokens_per_rank"], tpr)
    assert np.array_equal(got["expert_offset"], eo)
    bad = bool(((idx < -1) | (idx >= E)).any())
    assert bool(got["status"] & oracle.ST_BAD_INDEX) == bad


@pytest.mark.parametrize("R,T,K,E", [(1, 2, 2, 2), (2, 1, 2, 2), (2, 2, 1, 4), (1, 3, 2, 2),
                                     (2, 1, 3, 2)])
def test_layout_every_routing_of_tiny_shapes(R, T, K, E):
    values = list(range(-1, E))
    for combo in itertools.product(values, repeat=R * T * K):
        _check_layout(R, T, K, E, T, combo, align=1 + (sum(combo) % 3))


def test_layout_random_small_routings_with_bad_indices():
    r = np.random.default_rng(7)
    for _ in range(300):
        R = int(r.integers(1, 4))
        L = int(r.integers(1, 4))
        E, T, K = R * L, int(r.integers(0, 5)), int(r.integers(1, 4))
        idx = r.integers(-3, E + 2, size=(R * T, K))
        _check_layout(R, T, K, E, max(T, 1), idx, align=int(r.integers(1, 5)))


def test_layout_a5_worked_example():
    """The Ascend 950 table: 8 ranks x 8 local experts, 24 rows each, 192 per rank."""
    rows = [l.split() for l in open(os.path.join(GOLDEN, "a5_950_fused_counts.txt"))
            if l.strip() and not l.startswith("#")]
    want = np.array([[int(c) for c in r[2].split(",")] for r in rows])
    sums = np.array([int(r[3]) for r in rows])
    R, T, K, E = 8, 32, 6, 64
    n = np.arange(R * T)[:, None]
    idx = (n * K + np.arange(K)[None, :]) % E
    got = oracle.layout(R, T, K, E, T, idx)
    per_rank = got["recv_count"].reshape(R, E // R)
    assert np.array_equal(per_rank, want)
    assert np.array_equal(per_rank.sum(axis=1), sums)
    assert got["status"] == 0


@pytest.mark.parametrize("name", list(synth.WORKLOADS))
def test_layout_invariants_on_workload_routing(name):
    w = synth.workload(name)
    if w["N"] > 20000:
        w = synth.workload(name, T=max(1, 20000 // w["R"]))
    idx, _ = synth.make_routing(w)
    got = oracle.layout(w["R"], w["T"], w["K"], w["E"], w["M"], idx, layout=w["layout"])
    valid = (idx >= 0) & (idx < w["E"])
    assert got["recv_count"].sum() == valid.sum()
    assert np.array_equal(got["tokens_per_expert"].sum(axis=0), got["recv_count"])
    # each expert's slots are exactly 0 .. count-1, in (token, k) order
    s = got["token_slot"]
    for e in range(w["E"]):
        sel = np.nonzero(idx.reshape(-1) == e)[0]
        assert np.array_equal(s.reshape(-1)[sel], np.arange(sel.size))
    # a token with at least one expert is in at least one rank
    assert np.array_equal(got["is_token_in_rank"].any(axis=1), valid.any(axis=1))


def test_layout_capacity_overflow_flag():
    # duplicates inside a token can exceed cap = R*M in the padded layout
    R, T, K, E, M = 1, 2, 3, 2, 2
    idx = np.zeros((2, 3), np.int64)
    got = oracle.layout(R, T, K, E, M, idx, layout="padded")
    assert got["status"] & oracle.ST_CAPACITY
    assert list(got["token_slot"].reshape(-1)) == [0, 1, 2, 3, 4, 5]


# ---------------------------------------------------------------------------
# dispatch / combine / combine-backward
# ---------------------------------------------------------------------------

def _small(name, **kw):
    w = synth.workload(name, **kw)
    idx, wt = synth.make_routing(w)
    x = synth.make_x(w)
    return w, idx, wt, x


def _run_layout(w, idx, layout, align=1):
    return oracle.layout(w["R"], w["T"], w["K"], w["E"], w["M"], idx, layout=layout, align=align)


@pytest.mark.parametrize("layout,align", [("padded", 1), ("packed", 1), ("packed", 8)])
@pytest.mark.parametrize("shape", [{}, dict(R=4, T=5, M=8, K=3, E=8, H=64)],
                         ids=["one-rank", "four-ranks"])
def test_dispatch_bf16_is_an_exact_scatter(layout, align, shape):
    w, idx, wt, x = _small("tiny", **shape)
    lay = _run_layout(w, idx, layout, align)
    out = oracle.dispatch(w["R"], w["T"], w["K"], w["E"], w["M"], w["H"], "bf16", x, idx,
                          lay["token_slot"], lay["expert_offset"], topk_weights=wt,
                          layout=layout, align=align)
    rows_seen = np.zeros(out["recv_data"].shape[0], bool)
    for n in range(w["N"]):
        for k in range(w["K"]):
            e = idx[n, k]
            if e < 0:
                continue
            row = int(oracle.row_index(layout, w["R"], w["M"], e, lay["token_slot"][n, k],
                                       lay["expert_offset"]))
            rows_seen[row] = True
            assert np.array_equal(out["recv_data"][row].view(np.uint16), x[n])
            assert out["src_info"][row] == (n // w["T"]) * w["M"] + n % w["T"]
            assert out["recv_weights"][row] == wt[n, k]
    assert np.all(out["recv_data"][~rows_seen] == 0xAB)
    assert rows_seen.sum() == (idx >= 0).sum()


def test_combine_one_hot_identity_reproduces_x():
    w, idx, wt, x = _small("tiny")
    lay = _run_layout(w, idx, "padded")
    d = oracle.dispatch(w["R"], w["T"], w["K"], w["E"], w["M"], w["H"], "bf16", x, idx,
                        lay["token_slot"])
    y = d["recv_data"].view(np.uint16)  # identity experts
    valid = idx >= 0
    first = np.argmax(valid, axis=1)
    onehot = np.zeros_like(wt)
    onehot[np.arange(w["N"]), first] = 1.0
    out, st = oracle.combine(w["R"], w["T"], w["K"], w["E"], w["M"], w["H"], y, idx, onehot,
                             lay["token_slot"])
    has = valid.any(axis=1)
    assert st == 0
    assert np.array_equal(out[has], x[has])
    assert not out[~has].any()  # all-masked tokens give +0


def test_combine_equal_weights_identical_rows_is_exact():
    # K = 8 rows all equal to x, weights 1/8: every fma is exact, so the sum is x.
    H, K = 256, 8
    x = _bf16_row(H, seed=3)
    yrows = np.tile(x, (K, 1))
    out = oracle.combine_row(yrows, np.full(K, 0.125, np.float32), np.ones(K, np.uint8))
    assert np.array_equal(out, x)
    # and with weights 0.5 on two valid rows out of 8
    v = np.zeros(K, np.uint8)
    v[[2, 5]] = 1
    out = oracle.combine_row(yrows, np.full(K, 0.5, np.float32), v)
    assert np.array_equal(out, x)


def _bf16_ulp_distance(a, b):
    """Distance in bf16 ulps between two arrays of bf16 bits (monotone integer map)."""
    def key(u):
        u = u.astype(np.int64)
        return np.where(u & 0x8000, -(u & 0x7FFF), u)
    return np.abs(key(a) - key(b))


@pytest.mark.parametrize("seed", range(3))
def test_combine_within_one_ulp_of_float64_sum(seed):
    r = np.random.default_rng(seed)
    H, K = 2048, 8
    yrows = synth.to_bf16_bits(r.standard_normal((K, H)).astype(np.float32))
    wts = r.random(K).astype(np.float32)
    valid = (r.random(K) < 0.8).astype(np.uint8)
    out = oracle.combine_row(yrows, wts, valid)
    exact = (wts.astype(np.float64)[:, None] * oracle.bf16_to_f32(yrows) * valid[:, None]).sum(0)
    want = synth.to_bf16_bits(exact.astype(np.float32))  # float64 -> nearest fp32 -> bf16
    assert _bf16_ulp_distance(out, want).max() <= 1


def test_combine_backward_unweighted_equals_mxfp8_dispatch():
    w = synth.workload("prefill", R=4, T=24, E=32)
    idx, wt = synth.make_routing(w)
    pool, off = synth.g_source(w)
    g = synth.windows(pool, off, w["H"])
    lay = _run_layout(w, idx, "packed")
    args = (w["R"], w["T"], w["K"], w["E"], w["M"], w["H"])
    bwd = oracle.combine_bwd(*args, g, idx, wt, lay["token_slot"], lay["expert_offset"],
                             layout="packed", unweighted=True)
    dis = oracle.dispatch(*args, "mxfp8", g, idx, lay["token_slot"], lay["expert_offset"],
                          layout="packed")
    rows = lay["expert_offset"][-1]
    assert np.array_equal(bwd["grad_data"][:rows], dis["recv_data"][:rows])
    assert np.array_equal(bwd["grad_scale"][:rows], dis["recv_scale"][:rows])


def test_combine_backward_weighted_rows():
    w = synth.workload("prefill", R=2, T=16, E=16, H=256)
    idx, wt = synth.make_routing(w)
    pool, off = synth.g_source(w)
    g = synth.windows(pool, off, w["H"])
    lay = _run_layout(w, idx, "packed")
    bwd = oracle.combine_bwd(w["R"], w["T"], w["K"], w["E"], w["M"], w["H"], g, idx, wt,
                             lay["token_slot"], lay["expert_offset"], layout="packed")
    gf = oracle.bf16_to_f32(g)
    for n in range(w["N"]):
        for k in range(w["K"]):
            if idx[n, k] < 0:
                continue
            row = lay["expert_offset"][idx[n, k]] + lay["token_slot"][n, k]
            p = (np.float32(wt[n, k]) * gf[n]).astype(np.float32)  # one fp32 multiply each
            d, s = oracle.quant_row("mxfp8", p)
            assert np.array_equal(bwd["grad_data"][row], d)
            assert np.array_equal(bwd["grad_scale"][row], s)
            # dequantised grad is w * g within the e4m3 step
            X = s.astype(np.int64) - 127
            dec = oracle.e4m3_decode(d).astype(np.float64).reshape(-1, 32) * np.ldexp(1.0, X)[:, None]
            ref = p.astype(np.float64).reshape(-1, 32)
            assert np.all(np.abs(dec - ref) <= np.maximum(np.abs(ref) * 2 ** -4,
                                                          np.ldexp(2.0 ** -10, X)[:, None]))


# ---------------------------------------------------------------------------
# dequantisation and the combine of quantised expert outputs
# ---------------------------------------------------------------------------

def test_dequant_rows_worked_by_hand():
    # int8: codes times the row scale
    d = np.array([1, 0xFE, 127, 0x81], np.uint8)           # 1, -2, 127, -127
    s = np.float32([0.5]).view(np.uint8)
    assert list(oracle.dequant_row("int8_token", d, s, 4)) == [0.5, -1.0, 63.5, -63.5]
    # e4m3 per 128: 0x38 = 1.0, 0x40 = 2.0, 0xB8 = -1.0; scale_inv 2
    d = np.zeros(128, np.uint8)
    d[:3] = [0x38, 0x40, 0xB8]
    s = np.float32([2.0]).view(np.uint8)
    assert list(oracle.dequant_row("e4m3_b128", d, s, 128)[:3]) == [2.0, 4.0, -2.0]
    # MXFP8: byte 128 -> 2^1
    d = np.zeros(32, np.uint8)
    d[:2] = [0x38, 0x7E]                                      # 1.0, 448
    assert list(oracle.dequant_row("mxfp8", d, np.uint8([128]), 32)[:2]) == [2.0, 896.0]
    # MXFP4: element 0 is the low nibble; byte 126 -> 2^-1
    d = np.zeros(16, np.uint8)
    d[0] = 0x72                                               # low 2 (1.0), high 7 (6.0)
    assert list(oracle.dequant_row("mxfp4", d, np.uint8([126]), 32)[:2]) == [0.5, 3.0]


@pytest.mark.parametrize("mode", ["int8_token", "e4m3_b128", "mxfp8", "mxfp4"])
def test_dequant_of_quant_within_format_bounds(mode):
    H = 1024
    x = _bf16_row(H, seed=21)
    d, s = oracle.quant_row(mode, x)
    y = oracle.dequant_row(mode, d, s, H).astype(np.float64)
    xf = _f(x)
    if mode == "int8_token":
        sinv = float(s.view(np.float32)[0])
        assert np.all(np.abs(xf - y) <= 0.5 * sinv * (1 + 2 ** -20) + np.abs(xf) * 2 ** -21)
    elif mode == "e4m3_b128":
        sinv = np.repeat(s.view(np.float32).astype(np.float64), 128)
        assert np.all(np.abs(xf - y) <= np.maximum(np.abs(xf) * 2 ** -4, sinv * 2 ** -10) * (1 + 2 ** -18)
                      + np.abs(xf) * 2 ** -21)
    else:
        step = np.repeat(np.ldexp(1.0, s.astype(np.int64) - 127), 32)
        rel = 2 ** -4 if mode == "mxfp8" else 2 ** -1
        assert np.all(np.abs(xf - y) <= np.maximum(np.abs(xf) * rel, step * (2 ** -10 if mode == "mxfp8" else 0.25)))


def _table_dequant(mode, d, s, H):
    """Dequantisation written from the brute-force code tables of this file
    (not the oracle's decoders): exact values in float64."""
    if mode == "mxfp8":
        t = _e4m3_table()
        mag = t[d & 0x7F]
        v = np.where(d & 0x80, -mag, mag)
    else:
        t = _e2m1_table()
        codes = np.stack([d & 0xF, d >> 4], axis=1).reshape(-1)
        mag = t[codes & 0x7]
        v = np.where(codes & 0x8, -mag, mag)
    return v * np.repeat(np.ldexp(1.0, s.astype(np.int64) - 127), 32)


@pytest.mark.parametrize("mode", ["mxfp8", "mxfp4"])
def test_combine_of_mx_rows_equals_bf16_combine_of_their_values(mode):
    # An MX value (<= 4 significant bits times a power of two) is exact in
    # bf16, so the combine of quantised rows must equal the bf16 combine of the
    # decoded rows, bit for bit.
    r = np.random.default_rng(4)
    N, K, H = 6, 5, 256
    x = synth.to_bf16_bits((r.standard_normal((N * K, H)) * 3).astype(np.float32))
    D, S = oracle.row_bytes(mode, H)
    data = np.zeros((N, K, D), np.uint8)
    scale = np.zeros((N, K, S), np.uint8)
    dec = np.zeros((N, K, H), np.uint16)
    for i in range(N * K):
        d, s = oracle.quant_row(mode, x[i])
        data.reshape(-1, D)[i], scale.reshape(-1, S)[i] = d, s
        dec.reshape(-1, H)[i] = synth.to_bf16_bits(_table_dequant(mode, d, s, H).astype(np.float32))
    w = r.random((N, K)).astype(np.float32)
    valid = (r.random((N, K)) < 0.8).astype(np.uint8)
    got = oracle.combine_gathered_q(mode, data, scale, w, valid, H)
    want = oracle.combine_gathered(dec, w, valid)
    assert np.array_equal(got, want)


def test_combine_of_int8_rows_within_one_ulp_of_float64():
    r = np.random.default_rng(6)
    N, K, H = 4, 6, 512
    data = r.integers(0, 256, (N, K, H), dtype=np.uint8)
    sc = (r.random((N, K)) * 0.05 + 1e-3).astype(np.float32)
    w = r.random((N, K)).astype(np.float32)
    valid = np.ones((N, K), np.uint8)
    got = oracle.combine_gathered_q("int8_token", data, sc.view(np.uint8).reshape(N, K, 4), w, valid, H)
    q = data.view(np.int8).astype(np.float64)
    ref = (w.astype(np.float64)[:, :, None] * q * sc.astype(np.float64)[:, :, None]).sum(axis=1)
    want = synth.to_bf16_bits(ref.astype(np.float32))
    assert _bf16_ulp_distance(got, want).max() <= 1


def test_combine_of_bf16_rows_is_the_plain_combine():
    r = np.random.default_rng(8)
    N, K, H = 3, 4, 128
    y = synth.to_bf16_bits(r.standard_normal((N, K, H)).astype(np.float32))
    w = r.random((N, K)).astype(np.float32)
    valid = np.ones((N, K), np.uint8)
    got = oracle.combine_gathered_q("bf16", y.view(np.uint8).reshape(N, K, 2 * H), np.zeros((N, K, 0), np.uint8), w, valid, H)
    assert np.array_equal(got, oracle.combine_gathered(y, w, valid))


# ---------------------------------------------------------------------------
# E4M3 per 128 with round_scale (power-of-two fp32 scales) and with UE8M0
# (the same scales as e8m0 bytes, four to an int32)
# ---------------------------------------------------------------------------

def _block_max_in_every_32(x_bits):
    """bf16 row whose four 32-element sub-blocks of each 128-block share the
    128-block's maximum magnitude (its element 0 carries it, sign kept)."""
    xf = _f(x_bits).reshape(-1, 128).copy()
    amax = np.abs(xf).max(axis=1)
    for j in range(4):
        xf[:, 32 * j] = np.where(xf[:, 32 * j] < 0, -amax, amax)
    return synth.to_bf16_bits(xf.reshape(-1).astype(np.float32))


@pytest.mark.parametrize("seed", range(4))
def test_round_scale_equals_mxfp8_when_sub_blocks_share_the_maximum(seed):
    """With qmax 448, a 128-block whose four 32-blocks have the same maximum is
    quantised by round_scale exactly as MXFP8 quantises each of them (MXFP8 is
    pinned on its own above): the same codes, and 2^X = 2^(byte - 127)."""
    H = 1024
    x = _block_max_in_every_32(_bf16_row(H, scale=10.0 ** (seed - 2), seed=40 + seed))
    d2, s2 = oracle.quant_row("e4m3_b128_p2", x)
    dm, sm = oracle.quant_row("mxfp8", x)
    assert np.array_equal(d2, dm)
    p2 = s2.view(np.float32).astype(np.float64)
    assert np.array_equal(np.repeat(p2, 4), np.ldexp(1.0, sm.astype(np.int64) - 127))


@pytest.mark.parametrize("qmax", [448.0, 240.0, 127.0])
@pytest.mark.parametrize("seed", range(3))
def test_round_scale_is_the_smallest_power_of_two_that_fits(qmax, seed):
    """By definition: scale_inv = 2^X with amax * 2^-X <= qmax < amax * 2^-(X-1)
    (checked in float64 on the fp32 quotient), and the codes are e4m3 of x * 2^-X."""
    H = 2048
    x = _bf16_row(H, scale=10.0 ** (seed - 1), seed=50 + seed)
    d, s = oracle.quant_row("e4m3_b128_p2", x, e4m3_qmax=qmax)
    sinv = s.view(np.float32).astype(np.float64)
    X = np.log2(sinv)
    assert np.all(X == np.round(X))
    xf = _f(x).reshape(-1, 128)
    amax = np.abs(xf).max(axis=1)
    v = (amax.astype(np.float32) / np.float32(qmax)).astype(np.float64)
    assert np.all(v <= sinv) and np.all(v > sinv / 2)
    want = oracle.e4m3_encode((xf * (1.0 / sinv)[:, None]).astype(np.float32).reshape(-1))
    assert np.array_equal(d, want)


@pytest.mark.parametrize("H", [128, 384, 1024, 7168])
def test_ue8m0_is_round_scale_with_byte_scales(H):
    x = _bf16_row(H, seed=H)
    d2, s2 = oracle.quant_row("e4m3_b128_p2", x)
    du, su = oracle.quant_row("e4m3_b128_ue8m0", x)
    nb = H // 128
    assert oracle.row_bytes("e4m3_b128_ue8m0", H) == (H, 4 * ((nb + 3) // 4))
    assert np.array_equal(d2, du)
    X = np.log2(s2.view(np.float32).astype(np.float64)).astype(np.int64)
    assert np.array_equal(su[:nb].astype(np.int64), X + 127)
    assert np.all(su[nb:] == 0)
    # the two scale forms dequantise to the same values
    y2 = oracle.dequant_row("e4m3_b128_p2", d2, s2, H)
    yu = oracle.dequant_row("e4m3_b128_ue8m0", du, su, H)
    assert np.array_equal(y2.view(np.uint32), yu.view(np.uint32))


def test_round_scale_zero_block_uses_unit_scale():
    x = np.zeros(256, np.uint16)
    x[128:] = synth.to_bf16_bits(np.float32([3.0] * 128))
    d, s = oracle.quant_row("e4m3_b128_p2", x)
    assert list(s.view(np.float32)) == [1.0, 2.0 ** -7]     # 3/448 -> X = -7
    du, su = oracle.quant_row("e4m3_b128_ue8m0", x)
    assert list(su) == [127, 120, 0, 0]
    assert np.all(d[:128] == 0) and np.all(d[128:] == oracle.e4m3_encode(np.float32([3.0 * 128]))[0])


# ---------------------------------------------------------------------------
# non-finite inputs: an infinite block maximum, NaN elements, int8 NaN products
# ---------------------------------------------------------------------------

def test_infinite_block_maximum_takes_the_largest_exponent():
    """ceil(log2(inf)) clamped to the e8m0 range is 127: the infinite element
    saturates, every finite one falls to (signed) zero."""
    assert oracle.mx_exponent(np.float32([np.inf]), 448.0)[0] == 127
    assert oracle.mx_exponent(np.float32([np.inf]), 6.0)[0] == 127
    x = np.zeros(64, np.float32)
    x[3], x[4], x[5] = np.inf, -np.inf, -3.0
    x[40] = 1.5
    d, s = oracle.quant_row("mxfp8", x)
    assert list(s) == [254, 127 + oracle.mx_exponent(np.float32([1.5]), 448.0)[0]]
    assert list(d[3:6]) == [0x7E, 0xFE, 0x80] and np.all(d[[0, 1, 2, 6]] == 0)
    d, s = oracle.quant_row("mxfp4", x)
    # element 2i is the low nibble: byte 1 = (inf -> 6 | 0), byte 2 = (-inf -> -6 | -3 -> -0)
    assert s[0] == 254 and d[1] == (0x7 << 4) | 0x0 and d[2] == (0x8 << 4) | 0xF
    d, s = oracle.quant_row("e4m3_b128_p2", np.concatenate([x, np.zeros(64, np.float32)]))
    assert s.view(np.float32)[0] == np.float32(2.0 ** 127) and d[3] == 0x7E


def test_block_maximum_leaves_nan_out():
    r = np.random.default_rng(3)
    x = r.standard_normal(256).astype(np.float32)
    y = x.copy()
    y[[7, 100, 200]] = [np.nan, -np.nan, np.nan]
    z = x.copy()
    z[[7, 100, 200]] = 0.0
    for mode in ("mxfp8", "e4m3_b128", "e4m3_b128_p2", "int8_token"):
        dy, sy = oracle.quant_row(mode, y)
        dz, sz = oracle.quant_row(mode, z)
        assert np.array_equal(sy, sz), mode           # the scales ignore the NaNs
        keep = np.ones(256, bool)
        keep[[7, 100, 200]] = False
        assert np.array_equal(dy[keep], dz[keep]), mode
        want = 0x00 if mode == "int8_token" else 0x7F  # int8 has no NaN
        assert np.all(dy[[7, 100, 200]] == want), mode


def test_e2m1_infinities_saturate_and_nan_has_no_code():
    """satfinite clamps every overflow, infinities included, to +-6; the format
    has no NaN, so a NaN input has no specified code (the encoder's marker)."""
    got = oracle.e2m1_encode(np.float32([np.inf, -np.inf, 7.0, -1e30, np.nan, -np.nan]))
    assert list(got) == [0x7, 0xF, 0x7, 0xF, 0xFF, 0xFF]


def test_mxfp4_nan_elements_leave_the_rest_of_the_block_alone():
    """In an MXFP4 row the NaN elements stay out of the block maximum, so the
    scales and every other element's nibble equal those of the row with the
    NaNs replaced by zero (the NaN elements' own nibbles are unspecified)."""
    x = (np.random.default_rng(3).standard_normal(256) * 4).astype(np.float32)
    y = x.copy()
    y[[7, 100, 200, 201]] = np.nan
    z = x.copy()
    z[[7, 100, 200, 201]] = 0.0
    dy, sy = oracle.quant_row("mxfp4", y)
    dz, sz = oracle.quant_row("mxfp4", z)
    assert np.array_equal(sy, sz)
    nib_y = np.stack([dy & 0xF, dy >> 4], axis=1).reshape(-1)
    nib_z = np.stack([dz & 0xF, dz >> 4], axis=1).reshape(-1)
    keep = np.ones(256, bool)
    keep[[7, 100, 200, 201]] = False
    assert np.array_equal(nib_y[keep], nib_z[keep])


def test_int8_nan_products_are_zero():
    d, s = oracle.quant_row("int8_token", np.float32([np.inf, 1.0, -2.0, np.nan]))
    assert list(d) == [0, 0, 0, 0] and s.view(np.float32)[0] == np.inf


# ---------------------------------------------------------------------------
# weight gradient of the combine: dw[n,k] = <g[n,:], y[row(n,k),:]>
# ---------------------------------------------------------------------------

def _wgrad_case(layout="padded", align=1, H=32, seed=0):
    w = synth.workload("tiny", R=2, T=5, M=6, K=3, E=4, H=H)
    idx, _ = synth.make_routing(w, seed)
    idx[1, 2] = -1
    lay = _run_layout(w, idx, layout, align)
    rows = oracle.rows_max(w["R"], w["T"], w["K"], w["E"], w["M"], layout, align)
    r = np.random.default_rng(seed)
    # bf16 values with few significant bits: every double sum below is exact
    y = synth.to_bf16_bits((r.integers(-64, 64, (rows, H)) / 16.0).astype(np.float32))
    g = synth.to_bf16_bits((r.integers(-64, 64, (w["N"], H)) / 32.0).astype(np.float32))
    return w, idx, lay, y, g


@pytest.mark.parametrize("layout,align", [("padded", 1), ("packed", 1), ("packed", 4)])
def test_wgrad_equals_exact_rational_dot_products(layout, align):
    from fractions import Fraction
    w, idx, lay, y, g = _wgrad_case(layout, align)
    dw, st = oracle.combine_wgrad(w["R"], w["T"], w["K"], w["E"], w["M"], w["H"], g, y, idx,
                                  lay["token_slot"], lay["expert_offset"], layout=layout)
    assert st == 0
    gf, yf = _f(g), _f(y)
    for n in range(w["N"]):
        for k in range(w["K"]):
            if idx[n, k] < 0:
                assert dw[n, k] == 0.0
                continue
            row = int(oracle.row_index(layout, w["R"], w["M"], idx[n, k], lay["token_slot"][n, k],
                                       lay["expert_offset"]))
            exact = sum(Fraction(float(a)) * Fraction(float(b)) for a, b in zip(gf[n], yf[row]))
            assert dw[n, k] == np.float32(float(exact)), (n, k)


def test_wgrad_one_hot_gradient_picks_the_expert_value():
    w, idx, lay, y, g = _wgrad_case(H=64, seed=3)
    for j in (0, 17, 63):
        g1 = np.zeros_like(g)
        g1[:, j] = synth.to_bf16_bits(np.float32([1.0]))[0]
        dw, _ = oracle.combine_wgrad(w["R"], w["T"], w["K"], w["E"], w["M"], w["H"], g1, y, idx,
                                     lay["token_slot"], lay["expert_offset"])
        for n in range(w["N"]):
            for k in range(w["K"]):
                if idx[n, k] >= 0:
                    row = int(oracle.row_index("padded", w["R"], w["M"], idx[n, k],
                                               lay["token_slot"][n, k]))
                    assert dw[n, k] == _f(y[row:row + 1, j])[0]


def test_wgrad_flags_bad_indices():
    w, idx, lay, y, g = _wgrad_case()
    bad = idx.copy()
    bad[0, 0] = w["E"]
    dw, st = oracle.combine_wgrad(w["R"], w["T"], w["K"], w["E"], w["M"], w["H"], g, y, bad,
                                  lay["token_slot"], lay["expert_offset"])
    assert st & oracle.ST_BAD_INDEX and dw[0, 0] == 0.0


def test_wgrad_gathered_equals_the_layout_form():
    w, idx, lay, y, g = _wgrad_case("packed", 2, seed=7)
    dw, _ = oracle.combine_wgrad(w["R"], w["T"], w["K"], w["E"], w["M"], w["H"], g, y, idx,
                                 lay["token_slot"], lay["expert_offset"], layout="packed")
    yr = np.zeros((w["N"], w["K"], w["H"]), np.uint16)
    valid = idx >= 0
    for n, k in zip(*np.nonzero(valid)):
        row = int(oracle.row_index("packed", w["R"], w["M"], idx[n, k], lay["token_slot"][n, k],
                                   lay["expert_offset"]))
        yr[n, k] = y[row]
    dg, mag = oracle.combine_wgrad_gathered(g, yr, valid)
    assert np.array_equal(dg, dw)
    assert np.all(mag >= np.abs(dg)) and np.all(mag[~valid] == 0)


# ---------------------------------------------------------------------------
# the experts between dispatch and combine: per-expert linear maps
# ---------------------------------------------------------------------------

def test_expert_gemm_identity_weights_copy_the_rows():
    r = np.random.default_rng(1)
    E, H = 3, 64
    cnt = np.array([5, 0, 7], np.int64)
    eo = np.array([0, 8, 8, 16], np.int64)
    x = synth.to_bf16_bits(r.standard_normal((16, H)).astype(np.float32))
    w = np.zeros((E, H, H), np.uint16)
    one = synth.to_bf16_bits(np.float32([1.0]))[0]
    for e in range(E):
        w[e][np.arange(H), np.arange(H)] = one
    y = oracle.expert_gemm(x, w, eo[:E], cnt, H, y=np.full((16, H), 0x7777, np.uint16))
    for e in range(E):
        assert np.array_equal(y[eo[e]:eo[e] + cnt[e]], x[eo[e]:eo[e] + cnt[e]])
    assert np.all(y[5:8] == 0x7777) and np.all(y[15] == 0x7777)   # rows past count untouched


def test_expert_gemm_equals_exact_rational_products():
    from fractions import Fraction
    r = np.random.default_rng(2)
    E, H, N = 2, 32, 8
    cnt = np.array([3, 2], np.int64)
    eo = np.array([0, 4], np.int64)
    x = synth.to_bf16_bits((r.integers(-64, 64, (6, H)) / 16.0).astype(np.float32))
    w = synth.to_bf16_bits((r.integers(-64, 64, (E, N, H)) / 64.0).astype(np.float32))
    y = oracle.expert_gemm(x, w, eo, cnt, N)
    xf, wf = _f(x), _f(w)
    for e in range(E):
        for i in range(cnt[e]):
            row = eo[e] + i
            for j in range(N):
                exact = sum(Fraction(float(a)) * Fraction(float(b)) for a, b in zip(xf[row], wf[e, j]))
                want = synth.to_bf16_bits(np.float32([float(exact)]))[0]
                assert y[row, j] == want, (e, i, j)


# the same maps on MXFP8 operands (e4m3 codes, e8m0 scale per 32)
def _mx_operands(r, shape, lo=120, hi=134):
    """Seeded e4m3 codes (NaN codes 0x7F / 0xFF replaced by zero) and e8m0
    scale bytes in [lo, hi) for a [..., H] operand."""
    c = r.integers(0, 256, shape).astype(np.uint8)
    c[(c & 0x7F) == 0x7F] = 0
    s = r.integers(lo, hi, shape[:-1] + (shape[-1] // 32,)).astype(np.uint8)
    return c, s


def _mx_values(c, s):
    """Dequantised values, written out here from the e4m3 decoder and 2^(s-127)."""
    v = oracle.e4m3_decode(c).astype(np.float64)
    return v * np.ldexp(1.0, np.repeat(s.astype(np.int64) - 127, 32, axis=-1))


def test_expert_gemm_mx_identity_weights_give_the_dequantised_rows():
    r = np.random.default_rng(3)
    E, H = 2, 64
    cnt = np.array([3, 4], np.int64)
    eo = np.array([0, 4, 8], np.int64)
    xc, xs = _mx_operands(r, (8, H))
    wc = np.zeros((E, H, H), np.uint8)
    for e in range(E):
        wc[e][np.arange(H), np.arange(H)] = 0x38            # e4m3 1.0
    ws = np.full((E, H, H // 32), 127, np.uint8)            # 2^0
    y = oracle.expert_gemm_mx(xc, xs, wc, ws, eo[:E], cnt, H, y=np.full((8, H), 0x7777, np.uint16))
    for e in range(E):
        for i in range(cnt[e]):
            row = eo[e] + i
            want = synth.to_bf16_bits(oracle.dequant_row("mxfp8", xc[row], xs[row], H))
            want[want == 0x8000] = 0                         # a sum of zero products is +0
            assert np.array_equal(y[row], want), (e, i)
    assert np.all(y[3] == 0x7777)                            # past expert 0's count


def test_expert_gemm_mx_equals_exact_rational_sums():
    from fractions import Fraction
    r = np.random.default_rng(4)
    E, H, N = 2, 64, 4
    cnt = np.array([2, 3], np.int64)
    eo = np.array([0, 2], np.int64)
    xc, xs = _mx_operands(r, (5, H), 118, 136)
    wc, ws = _mx_operands(r, (E, N, H), 118, 136)
    y = oracle.expert_gemm_mx(xc, xs, wc, ws, eo, cnt, N)
    xv, wv = _mx_values(xc, xs), _mx_values(wc, ws)
    for e in range(E):
        for i in range(cnt[e]):
            row = eo[e] + i
            for j in range(N):
                exact = sum(Fraction(float(a)) * Fraction(float(b)) for a, b in zip(xv[row], wv[e, j]))
                want = synth.to_bf16_bits(np.float32([float(exact)]))[0]
                assert y[row, j] == want, (e, i, j)


def test_expert_gemm_mx_equals_bf16_maps_on_dequantised_operands():
    """e4m3 values times powers of two in the normal range are bf16 values, so
    the MX maps equal the (separately pinned) bf16 maps of the dequantised
    operands, bit for bit."""
    r = np.random.default_rng(5)
    E, H, N = 3, 256, 16
    cnt = np.array([4, 0, 6], np.int64)
    eo = np.array([0, 8, 8], np.int64)
    xc, xs = _mx_operands(r, (16, H))
    wc, ws = _mx_operands(r, (E, N, H))
    xb = synth.to_bf16_bits(_mx_values(xc, xs).astype(np.float32))
    wb = synth.to_bf16_bits(_mx_values(wc, ws).astype(np.float32))
    assert np.array_equal(oracle.bf16_to_f32(xb).astype(np.float64), _mx_values(xc, xs))
    want = oracle.expert_gemm(xb, wb, eo, cnt, N)
    got = oracle.expert_gemm_mx(xc, xs, wc, ws, eo, cnt, N)
    assert np.array_equal(got, want)


# the same maps on MXFP4 operands (packed e2m1 codes, e8m0 scale per 32)
def _fp4_operands(r, shape, lo=120, hi=134):
    """Seeded packed e2m1 codes (two a byte) and e8m0 scales for a [..., H] operand."""
    c = r.integers(0, 256, shape[:-1] + (shape[-1] // 2,)).astype(np.uint8)
    s = r.integers(lo, hi, shape[:-1] + (shape[-1] // 32,)).astype(np.uint8)
    return c, s


def _fp4_values(c, s):
    """Dequantised values written out here: e2m1 table, even element in the low nibble."""
    table = oracle.e2m1_decode(np.arange(16, dtype=np.uint8)).astype(np.float64)
    v = np.empty(c.shape[:-1] + (2 * c.shape[-1],), np.float64)
    v[..., 0::2] = table[c & 0xF]
    v[..., 1::2] = table[c >> 4]
    return v * np.ldexp(1.0, np.repeat(s.astype(np.int64) - 127, 32, axis=-1))


def test_expert_gemm_mxfp4_identity_weights_give_the_dequantised_rows():
    r = np.random.default_rng(6)
    E, H = 2, 64
    cnt = np.array([3, 4], np.int64)
    eo = np.array([0, 4, 8], np.int64)
    xc, xs = _fp4_operands(r, (8, H))
    wc = np.zeros((E, H, H // 2), np.uint8)
    for e in range(E):
        for j in range(H):
            wc[e, j, j // 2] = 0x2 if j % 2 == 0 else 0x20        # e2m1 1.0 at element j
    ws = np.full((E, H, H // 32), 127, np.uint8)
    y = oracle.expert_gemm_mxfp4(xc, xs, wc, ws, eo[:E], cnt, H, y=np.full((8, H), 0x7777, np.uint16))
    for e in range(E):
        for i in range(cnt[e]):
            row = eo[e] + i
            want = synth.to_bf16_bits(oracle.dequant_row("mxfp4", xc[row], xs[row], H))
            want[want == 0x8000] = 0                                 # a sum of zero products is +0
            assert np.array_equal(y[row], want), (e, i)
    assert np.all(y[3] == 0x7777)


def test_expert_gemm_mxfp4_equals_exact_rational_sums():
    from fractions import Fraction
    r = np.random.default_rng(7)
    E, H, N = 2, 64, 4
    cnt = np.array([2, 3], np.int64)
    eo = np.array([0, 2], np.int64)
    xc, xs = _fp4_operands(r, (5, H), 118, 136)
    wc, ws = _fp4_operands(r, (E, N, H), 118, 136)
    y = oracle.expert_gemm_mxfp4(xc, xs, wc, ws, eo, cnt, N)
    xv, wv = _fp4_values(xc, xs), _fp4_values(wc, ws)
    for e in range(E):
        for i in range(cnt[e]):
            row = eo[e] + i
            for j in range(N):
                exact = sum(Fraction(float(a)) * Fraction(float(b)) for a, b in zip(xv[row], wv[e, j]))
                want = synth.to_bf16_bits(np.float32([float(exact)]))[0]
                assert y[row, j] == want, (e, i, j)


def test_expert_gemm_mxfp4_equals_bf16_maps_on_dequantised_operands():
    r = np.random.default_rng(8)
    E, H, N = 3, 256, 16
    cnt = np.array([4, 0, 6], np.int64)
    eo = np.array([0, 8, 8], np.int64)
    xc, xs = _fp4_operands(r, (16, H))
    wc, ws = _fp4_operands(r, (E, N, H))
    xb = synth.to_bf16_bits(_fp4_values(xc, xs).astype(np.float32))
    wb = synth.to_bf16_bits(_fp4_values(wc, ws).astype(np.float32))
    assert np.array_equal(oracle.bf16_to_f32(xb).astype(np.float64), _fp4_values(xc, xs))
    want = oracle.expert_gemm(xb, wb, eo, cnt, N)
    got = oracle.expert_gemm_mxfp4(xc, xs, wc, ws, eo, cnt, N)
    assert np.array_equal(got, want)


# ---------------------------------------------------------------------------
# the experts' gated MLP: GMM1 -> SwiGLU -> MXFP8 requant -> GMM2
# ---------------------------------------------------------------------------
# e to 60 digits (a textbook constant, so that no value below comes from a
# library exp routine)
_E_DIGITS = "2.718281828459045235360287471352662497757247093699959574966967"


def _silu_exact(a):
    """silu(a) = a / (1 + e^-a) for an integer or half-integer a, in 50-digit
    decimal arithmetic from the digits of e."""
    from decimal import Decimal, getcontext
    getcontext().prec = 50
    e = Decimal(_E_DIGITS)
    two_a = int(round(2 * a))
    assert two_a == 2 * a
    root = e.sqrt()                       # e^(1/2)
    p = root ** abs(two_a)                # e^|a|
    ema = (1 / p) if a > 0 else p         # e^-a
    return Decimal(two_a) / 2 / (1 + ema)


def _ffn_case(E, H, I, rows_per_e, gate_vals, up_vals, seed=0):
    """Operands whose GMM1 outputs are set by hand: every row's codes are 1.0
    at one position (scale 2^0), W1's gate row j of expert e holds gate_vals
    at that position and W1's up row j holds up_vals; W2 holds small integers."""
    enc = oracle.e4m3_encode
    rows = E * rows_per_e
    xc = np.zeros((rows, H), np.uint8)
    xc[:, 0] = enc(np.float32([1.0]))[0]
    xs = np.full((rows, H // 32), 127, np.uint8)
    w1c = np.zeros((E, 2 * I, H), np.uint8)
    w1c[:, :I, 0] = enc(np.asarray(gate_vals, np.float32))
    w1c[:, I:, 0] = enc(np.asarray(up_vals, np.float32))
    w1s = np.full((E, 2 * I, H // 32), 127, np.uint8)
    r = np.random.default_rng(seed)
    w2c = enc(r.integers(-3, 4, (E, H, I)).astype(np.float32))
    w2s = np.full((E, H, I // 32), 127, np.uint8)
    eo = np.arange(E, dtype=np.int64) * rows_per_e
    cnt = np.full(E, rows_per_e, np.int64)
    return xc, xs, w1c, w1s, w2c, w2s, eo, cnt


def _f32_ulp(v):
    return np.spacing(np.abs(np.float32(v)))


def test_ffn_silu_matches_the_constant_e_and_the_gate_up_order():
    """z = silu(gate) * up with gate the first I outputs of GMM1: each z is
    within one fp32 ulp of the 50-digit value; with the halves swapped the
    values would be silu(up) * gate, which differ."""
    from decimal import Decimal
    gates = [1.0, -1.0, 2.0, -2.0, 0.5, -0.5, 3.0, 4.0] * 4
    ups = [3.0, 3.0, 1.0, 1.0, 1.0, -2.0, 0.5, -1.0] * 4
    case = _ffn_case(1, 64, 32, 2, gates, ups)
    o = oracle.expert_ffn_mx(*case)
    for j in range(32):
        want = float(_silu_exact(gates[j]) * Decimal(ups[j]))
        got = float(o["z"][0, j])
        assert abs(got - want) <= _f32_ulp(want), (j, got, want)
    swapped = float(_silu_exact(ups[0]) * Decimal(gates[0]))
    assert abs(float(o["z"][0, 0]) - swapped) > 0.5


def test_ffn_silu_identities():
    """silu(0) = 0; silu(a) - silu(-a) = a; silu(a) = a for a large gate."""
    gates = [0.0, 5.0, -5.0, 7.0, -7.0, 448.0, 0.0, 1.5] * 4
    ups = [9.0, 1.0, 1.0, 1.0, 1.0, 3.0, -6.0, 1.0] * 4
    o = oracle.expert_ffn_mx(*_ffn_case(1, 64, 32, 1, gates, ups))
    z = o["z"][0].astype(np.float64)
    assert z[0] == 0.0 and z[6] == 0.0
    assert abs((z[1] - z[2]) - 5.0) <= 2 * _f32_ulp(5.0)
    assert abs((z[3] - z[4]) - 7.0) <= 2 * _f32_ulp(7.0)
    assert z[5] == 448.0 * 3.0                      # e^-448 is far below half an ulp


def test_ffn_zero_gate_gives_zero_codes_and_unit_scale():
    o = oracle.expert_ffn_mx(*_ffn_case(2, 64, 64, 3, [0.0] * 64, [5.0] * 64))
    assert np.all(o["z"] == 0) and np.all(o["zc"] == 0) and np.all(o["zs"] == 127)
    assert np.all(o["y"] == 0)


def _mxfp8_by_search(z):
    """MXFP8 of one fp32 row by brute force: per 32 elements the smallest
    power of two 2^X (X in [-127, 127]) with amax/448 <= 2^X, found by search,
    and the nearest e4m3 code of z * 2^-X (ties to the even code)."""
    z = np.asarray(z, np.float32)
    table = _e4m3_table()
    codes = np.empty(z.size, np.uint8)
    scales = np.empty(z.size // 32, np.uint8)
    for b in range(z.size // 32):
        blk = z[32 * b: 32 * b + 32]
        amax = float(np.max(np.abs(blk)))
        v = float(np.float32(amax) / np.float32(448.0))
        X = 0 if amax == 0 else next(x for x in range(-127, 128) if 2.0 ** x >= v)
        scales[b] = X + 127
        codes[32 * b: 32 * b + 32] = _brute_encode(blk.astype(np.float64) * 2.0 ** -X, table, 0x80)
    return codes, scales


def test_ffn_chain_equals_brute_force_on_small_integers():
    """Small-integer operands (every GMM1 output an exact integer): the oracle's
    h, z, requantised codes and scales and y equal a brute-force chain written
    here -- integer matmul, silu from the digits of e, MXFP8 by search, the
    second product summed exactly and rounded by torch."""
    from fractions import Fraction
    r = np.random.default_rng(7)
    E, H, I, per = 2, 64, 64, 3
    rows = E * per
    enc = oracle.e4m3_encode
    xi = r.integers(0, 4, (rows, H))
    w1i = r.integers(-1, 2, (E, 2 * I, H))
    w2i = r.integers(-2, 3, (E, H, I))
    xc = enc(xi.astype(np.float32))
    xs = np.full((rows, H // 32), 127, np.uint8)
    w1c, w1s = enc(w1i.astype(np.float32)), np.full((E, 2 * I, H // 32), 127, np.uint8)
    w2c, w2s = enc(w2i.astype(np.float32)), np.full((E, H, I // 32), 127, np.uint8)
    eo = np.arange(E, dtype=np.int64) * per
    cnt = np.full(E, per, np.int64)
    o = oracle.expert_ffn_mx(xc, xs, w1c, w1s, w2c, w2s, eo, cnt)
    table = _e4m3_table()
    for e in range(E):
        for rr in range(e * per, (e + 1) * per):
            h = w1i[e] @ xi[rr]                                  # exact integers
            assert np.array_equal(o["h"][rr], h.astype(np.float32))
            z = np.array([np.float32(float(_silu_exact(int(h[j])) * int(h[I + j])))
                          for j in range(I)], np.float32)
            assert np.array_equal(o["z"][rr], z), rr
            zc, zs = _mxfp8_by_search(z)
            assert np.array_equal(o["zc"][rr], zc) and np.array_equal(o["zs"][rr], zs), rr
            zv = [Fraction(float(table[c & 0x7F])) * (-1 if c & 0x80 else 1) *
                  Fraction(2) ** (int(zs[i // 32]) - 127) for i, c in enumerate(zc)]
            y = np.empty(H, np.float32)
            for j in range(H):
                y[j] = np.float32(float(sum(zv[i] * int(w2i[e, j, i]) for i in range(I))))
            want = torch.from_numpy(y).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
            assert np.array_equal(o["y"][rr], want), rr
    untouched = np.ones(rows, bool)
    untouched[:E * per] = False
    assert np.all(o["y"][untouched] == 0)


def test_ffn_requant_window_and_power_of_two_scales():
    """On random MX operands: each requantised block's scale is a power of two
    with the block maximum in (224, 448] after scaling, and every dequantised
    element lies within half an e4m3 step of z."""
    r = np.random.default_rng(11)
    E, H, I, per = 2, 128, 96, 4
    rows = E * per
    xc = r.integers(0, 0x7E, (rows, H)).astype(np.uint8)
    xs = r.integers(118, 126, (rows, H // 32)).astype(np.uint8)
    w1c = (r.integers(0, 0x7E, (E, 2 * I, H)) | (r.integers(0, 2, (E, 2 * I, H)) << 7)).astype(np.uint8)
    w1s = r.integers(116, 124, (E, 2 * I, H // 32)).astype(np.uint8)
    w2c = r.integers(0, 0x7E, (E, H, I)).astype(np.uint8)
    w2s = np.full((E, H, I // 32), 120, np.uint8)
    o = oracle.expert_ffn_mx(xc, xs, w1c, w1s, w2c, w2s, np.array([0, per]), np.array([per, per]))
    dec = oracle.e4m3_decode(o["zc"]).astype(np.float64)
    X = o["zs"].astype(np.int64) - 127
    for rr in range(rows):
        for b in range(I // 32):
            z = o["z"][rr, 32 * b: 32 * b + 32].astype(np.float64)
            q = dec[rr, 32 * b: 32 * b + 32] * 2.0 ** X[rr, b]
            amax = np.abs(z).max()
            if amax == 0:
                continue
            assert 224 < amax * 2.0 ** -X[rr, b] <= 448
            step = np.ldexp(1.0, np.floor(np.log2(np.maximum(np.abs(z) * 2.0 ** -X[rr, b], 2 ** -6))).astype(int) - 3)
            assert np.all(np.abs(q - z) <= 0.5 * step * 2.0 ** X[rr, b] + 2.0 ** (X[rr, b] - 10))
