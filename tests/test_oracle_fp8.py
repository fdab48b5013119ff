"""Pins of the fp8 backbone oracle (oracle/fp8.py): the E4M3 format of the OCP 8-bit floating point
specification, its round-to-nearest-even with saturation, and the per-row quantisation."""
import numpy as np

from oracle import fp8


def test_e4m3_table_known_values():
    v = fp8.E4M3_TABLE
    assert v[0x00] == 0.0 and v[0x38] == 1.0 and v[0x3C] == 1.5 and v[0x7E] == 448.0
    assert v[0x08] == 2.0 ** -6 and v[0x01] == 2.0 ** -9 and v[0x07] == 7 * 2.0 ** -9
    assert np.isnan(v[0x7F]) and np.isnan(v[0xFF]) and v[0xFE] == -448.0 and v[0xB8] == -1.0
    finite = v[~np.isnan(v)]
    assert len(finite) == 254 and np.max(finite) == 448.0
    pos = v[0x00:0x7F]
    assert np.all(np.diff(pos) > 0)  # codes 0..126 increase in value


def test_round_trip_of_every_finite_code():
    for c in range(256):
        if c in (0x7F, 0xFF, 0x80):
            continue
        assert int(fp8.e4m3_round(np.float32(fp8.E4M3_TABLE[c]))) == c
    assert int(fp8.e4m3_round(np.float32(-0.0))) in (0x00, 0x80)


def test_round_to_nearest_even_brute_force():
    rng = np.random.default_rng(8)
    x = np.concatenate([rng.standard_normal(4000) * 10 ** rng.uniform(-4, 2.5, 4000),
                        rng.uniform(-500, 500, 500)]).astype(np.float32)
    codes = fp8.e4m3_round(x)
    cand = np.arange(256)
    vals = fp8.E4M3_TABLE
    ok = ~np.isnan(vals)
    for xi, c in zip(x.astype(np.float64), codes):
        t = np.clip(xi, -448.0, 448.0)
        d = np.abs(vals[ok] - t)
        best = cand[ok][d == d.min()]
        best_vals = {vals[b] for b in best}
        assert vals[c] in best_vals or (vals[c] == 0 and 0.0 in best_vals)
        if len(best_vals) == 2:  # a tie: the even code
            assert c % 2 == 0


def test_midpoints_go_to_the_even_code_and_saturation():
    v = fp8.E4M3_TABLE
    for c in range(0, 0x7E):
        mid = np.float32((v[c] + v[c + 1]) / 2)
        if float(mid) != (v[c] + v[c + 1]) / 2:
            continue  # not representable in fp32
        got = int(fp8.e4m3_round(mid))
        assert got == (c if c % 2 == 0 else c + 1), c
    assert int(fp8.e4m3_round(np.float32(463.9))) == 0x7E
    assert int(fp8.e4m3_round(np.float32(1e6))) == 0x7E and int(fp8.e4m3_round(np.float32(-1e6))) == 0xFE
    assert int(fp8.e4m3_round(np.float32(2.0 ** -11))) == 0x00   # below half the smallest subnormal
    assert int(fp8.e4m3_round(np.float32(2.0 ** -10 * 1.01))) == 0x01


def test_quantize_rows_scale_and_error():
    rng = np.random.default_rng(9)
    w = (0.02 * rng.standard_normal((64, 512))).astype(np.float32)
    w[3] = 0.0
    codes, sc = fp8.quantize_rows(w)
    assert sc[3] == 1.0 and np.all(codes[3] % 0x80 == 0)
    wh = fp8.dequantize_rows(codes, sc)
    # the row maximum lands on +-448; every element within half a step of the E4M3 grid scaled
    assert np.all(np.abs(fp8.E4M3_TABLE[codes[np.arange(64) != 3].astype(np.int64)]).max(axis=1) == 448.0)
    rel = np.abs(wh - w) / np.maximum(np.abs(w), 2.0 ** -6 * sc[:, None])
    assert rel.max() <= 2.0 ** -4 + 1e-7


def test_library_fp8_quantiser_matches_oracle():
    import tenant_mixed_precision_b200 as dc
    rng = np.random.default_rng(10)
    w = np.concatenate([(0.02 * rng.standard_normal((40, 384))),
                        rng.standard_normal((8, 384)) * 10 ** rng.uniform(-6, 3, size=(8, 1))]).astype(np.float32)
    w[5] = 0.0
    w[7, :] = 1e-30  # subnormal scale region
    codes, sc = dc.dc_quantize_fp8_rows(w)
    oc, osc = fp8.quantize_rows(w)
    assert np.array_equal(sc, osc)
    # the same values (a code 0x80, minus zero, equals 0x00)
    assert np.array_equal(fp8.E4M3_TABLE[codes.astype(np.int64)], fp8.E4M3_TABLE[oc.astype(np.int64)])
    blob = dc.fp8_weight_blob(codes, sc)
    assert blob.nbytes == w.size + 4 * w.shape[0]


def test_backbone_is_the_plain_product_on_exact_inputs():
    """F3 pinned: when every row's largest magnitude is 448 times a power of two and every element is
    that power of two times an E4M3 value, the per-row/per-token scales are exact powers of two, the
    quantisation loses nothing, and the oracle's fp8 backbone equals the plain product W x^T (for a
    non-square W, so a transposed operand would show); `rows` selects output rows."""
    rng = np.random.default_rng(21)
    finite = fp8.E4M3_TABLE[np.arange(0x7F)]  # non-negative finite values, 0 .. 448

    def exact_rows(n, m, expo):
        v = rng.choice(finite, size=(n, m)) * rng.choice([-1.0, 1.0], size=(n, m))
        v[:, 0] = 448.0  # the row maximum
        return (v * (2.0 ** expo)[:, None]).astype(np.float32)

    W = exact_rows(24, 40, rng.integers(-12, 3, size=24))
    x = exact_rows(5, 40, rng.integers(-6, 6, size=5))
    wc, ws = fp8.quantize_rows(W)
    assert np.array_equal(fp8.dequantize_rows(wc, ws), W.astype(np.float64))
    got = fp8.backbone(wc, ws, x)
    want = x.astype(np.float64) @ W.astype(np.float64).T
    assert got.shape == (5, 24)
    assert np.array_equal(got, want)
    rows = np.array([3, 17, 0])
    assert np.array_equal(fp8.backbone(wc, ws, x, rows=rows), want[:, rows])
