"""Pins of the fp64 oracle against what the pages and mathematics fix (no GPU).

Each test names the property it checks and the passage the property comes from.  The pages print
no worked numeric example of the compression or of a forward pass, so the pins are closed forms,
invariants, brute force and hand-derived fixtures (tests/golden/).
"""
import math
import os

import numpy as np
import pytest

import oracle
from oracle.delta_come import _rtn_quantize_rows
from tenant_mixed_precision_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_rtn_golden():
    rows = []
    with open(os.path.join(GOLDEN, "rtn_groups.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            bits, vals, scale, zero, codes = [p.strip() for p in line.split("|")]
            rows.append((int(bits), [float(v) for v in vals.split(",")], float(scale), float(zero),
                         [int(c) for c in codes.split(",")]))
    return rows


# --------------------------------------------------------------------------------------------
# RTN (reading R1; "Approach" section of the Delta-CoMe summary page fixes the 8/3/2 widths)
# --------------------------------------------------------------------------------------------
@pytest.mark.parametrize("case", _read_rtn_golden())
def test_rtn_hand_derived_groups(case):
    bits, vals, scale, zero, codes = case
    c, s, z = oracle.rtn_quantize_group(np.array(vals), bits)
    assert s == scale
    assert z == zero
    assert list(c) == codes


def test_rtn_hand_groups_padded_to_128():
    # zeros never move lo/hi because 0 is forced into the range: padding a group to 128 with
    # zeros leaves the hand-derived codes of the leading elements unchanged
    for bits, vals, scale, zero, codes in _read_rtn_golden():
        g = np.zeros(128)
        g[: len(vals)] = vals
        c, s, z = oracle.rtn_quantize_group(g, bits)
        assert (s, z) == (scale, zero)
        assert list(c[: len(vals)]) == codes
        assert np.all(c[len(vals):] == int(zero))


def test_fp16_scale_rounding_is_single_rne():
    # a value just above a half-way point must round up (no double rounding through fp32)
    assert float(np.float16(1 + 2 ** -11 + 2 ** -40)) == 1 + 2 ** -10
    assert float(np.float16(1 + 2 ** -11)) == 1.0
    assert float(np.float16(1 + 3 * 2 ** -11)) == 1 + 2 ** -9


@pytest.mark.parametrize("bits", [2, 3, 8])
def test_rtn_brute_force_nearest_grid_point(bits):
    # For every element whose value lies inside the representable range, the code is the grid
    # point (c - zero) * scale nearest to v, found here by trying every code.
    rng = np.random.default_rng(100 + bits)
    qmax = (1 << bits) - 1
    for _ in range(50):
        g = rng.standard_normal(128) * rng.uniform(1e-3, 1.0)
        if rng.random() < 0.3:
            g = np.abs(g)
        c, s, z = oracle.rtn_quantize_group(g, bits)
        grid = (np.arange(qmax + 1) - z) * s
        for v, code in zip(g, c):
            d = np.abs(v - grid)
            best = np.flatnonzero(d == d.min())
            if v / s + z < -0.5 or v / s + z > qmax + 0.5:
                # outside the grid: clamped to the nearest end
                assert code in (0, qmax)
                continue
            assert code in best
            assert abs(v - (code - z) * s) <= s / 2 + 1e-15


@pytest.mark.parametrize("bits", [2, 3, 8, 16])
def test_rtn_codes_in_range_and_error_bound(bits):
    rng = np.random.default_rng(7 + bits)
    v = rng.standard_normal(1024) / 32.0
    q = oracle.rtn_quantize_vector(v, bits)
    qmax = (1 << bits) - 1
    assert q.codes.min() >= 0 and q.codes.max() <= qmax
    vh = oracle.dequantize_vector(q)
    g = np.arange(v.size) // 128
    unclamped = (q.codes > 0) & (q.codes < qmax)
    assert np.all(np.abs(v - vh)[unclamped] <= q.scales[g][unclamped] / 2 + 1e-15)
    # zero is an integer in range, so 0.0 is exactly on every grid
    assert np.all(q.zeros == np.round(q.zeros)) and q.zeros.min() >= 0 and q.zeros.max() <= qmax


@pytest.mark.parametrize("bits", [2, 3, 8])
@pytest.mark.parametrize("sign", [1.0, -1.0])
def test_rtn_one_sign_group_stays_on_the_grid(bits, sign):
    # A group whose values all have one sign: 0 is forced into the range (lo = min(0, min g),
    # hi = max(0, max g)), so the grid runs from 0 to the far end of the group and no element is
    # clipped by more than the fp16 rounding of the scale can move the grid's end:
    # |v - v_hat| <= scale / 2 + qmax * |scale - (hi - lo) / qmax|.
    rng = np.random.default_rng(300 + bits)
    qmax = (1 << bits) - 1
    for _ in range(40):
        g = sign * (np.abs(rng.standard_normal(128)) * rng.uniform(1e-4, 2.0) + rng.uniform(0, 0.5))
        c, s, z = oracle.rtn_quantize_group(g, bits)
        lo, hi = min(0.0, g.min()), max(0.0, g.max())
        assert z == (0.0 if sign > 0 else float(qmax)) or abs(z - (-lo / s)) <= 0.5 + 1e-12
        assert c.min() >= 0 and c.max() <= qmax
        slack = qmax * abs(s - (hi - lo) / qmax)
        err = np.abs(g - (c - z) * s)
        assert np.all(err <= s / 2 + slack + 1e-15)
        # the element farthest from 0 lands on the grid's far end (or one step in)
        far = int(np.argmax(np.abs(g)))
        assert c[far] in ((qmax, qmax - 1) if sign > 0 else (0, 1))


def test_rtn_vectorised_rows_match_group_loop():
    rng = np.random.default_rng(3)
    M = rng.standard_normal((5, 384)) * 0.05
    for bits in (2, 3, 8):
        c, s, z = _rtn_quantize_rows(M, bits)
        for i in range(5):
            q = oracle.rtn_quantize_vector(M[i], bits)
            assert np.array_equal(c[i], q.codes) and np.array_equal(s[i], q.scales) and np.array_equal(z[i], q.zeros)


def test_rtn_rejects_non_finite():
    with pytest.raises(ValueError):
        oracle.rtn_quantize_group(np.array([0.0, np.inf]), 2)


# --------------------------------------------------------------------------------------------
# SVD and Eckart-Young ("Delta-CoMe的技术原理": SVD of the delta; low-rank structure)
# --------------------------------------------------------------------------------------------
def test_svd_reconstructs_and_is_orthonormal():
    case = synth.single_linear_case(seed=0)
    D = oracle.delta_weights(case.w_base, case.w_ft[0])
    U, s, Vt = oracle.svd_factors(D)
    assert np.linalg.norm(U @ np.diag(s) @ Vt - D) / np.linalg.norm(D) < 1e-12
    assert np.abs(U.T @ U - np.eye(U.shape[1])).max() < 1e-12
    assert np.abs(Vt @ Vt.T - np.eye(Vt.shape[0])).max() < 1e-12
    assert np.all(np.diff(s) <= 0)
    # sign convention R4: the largest-magnitude entry of every v_i is positive
    j = np.argmax(np.abs(Vt), axis=1)
    assert np.all(Vt[np.arange(Vt.shape[0]), j] > 0)


def test_svd_recovers_constructed_long_tail_spectrum():
    # Delta = Q1 diag(s) Q2^T with orthonormal Q's: the SVD must return s exactly (to rounding)
    # and the Q columns up to sign.  Long-tail s_i = s0 i^-0.8 as in "Delta-CoMe的技术原理"
    # (most singular values small, a few large).
    rng = np.random.default_rng(1)
    d_out, d_in, r = 384, 256, 60
    q1 = synth.random_orthonormal(rng, d_out, r)
    q2 = synth.random_orthonormal(rng, d_in, r)
    s = 0.02 * math.sqrt(256) * np.arange(1, r + 1) ** -0.8
    U, sig, Vt = oracle.svd_factors((q1 * s) @ q2.T)
    assert np.max(np.abs(sig[:r] - s)) < 1e-13
    assert np.max(np.abs(sig[r:])) < 1e-13
    for i in range(r):
        assert abs(abs(np.dot(U[:, i], q1[:, i])) - 1) < 1e-9
        assert abs(abs(np.dot(Vt[i], q2[:, i])) - 1) < 1e-9


@pytest.mark.parametrize("k", [0, 1, 10, 42, 200, 511])
def test_eckart_young_tail(k):
    case = synth.single_linear_case(seed=0)
    D = oracle.delta_weights(case.w_base, case.w_ft[1])
    U, s, Vt = oracle.svd_factors(D)
    Dk = (U[:, :k] * s[:k]) @ Vt[:k]
    err = np.linalg.norm(D - Dk)
    assert abs(err - oracle.eckart_young_tail(s, k)) <= 1e-10 * np.linalg.norm(D)


def test_full_rank_high_bit_reconstruction():
    # all ranks kept at 16 bits reconstruct the delta within the RTN bound
    # sum_i S_i (|du_i| + |dv_i| + |du_i||dv_i|); with no quantisation at all the SVD alone
    # reconstructs to 1e-12 (previous test)
    rng = np.random.default_rng(5)
    d = 256
    D = (synth.random_orthonormal(rng, d, d) * (0.05 / np.arange(1, d + 1))) @ synth.random_orthonormal(rng, d, d).T
    U, s, Vt = oracle.svd_factors(D)
    a = oracle.compress_factors(U.astype(np.float32), s.astype(np.float32), Vt.astype(np.float32), [(16, d)])
    Uh, S, Vh = oracle.dequantized_factors(a)
    Dh = (Uh * S) @ Vh
    du = np.linalg.norm(Uh - U.astype(np.float32), axis=0)
    dv = np.linalg.norm(Vh - Vt.astype(np.float32), axis=1)
    bound = np.sum(S * (du + dv + du * dv))
    # fp32 rounding of the factors adds at most ~1e-7 relative
    Df = (U.astype(np.float32).astype(np.float64) * S) @ Vt.astype(np.float32).astype(np.float64)
    assert np.linalg.norm(Df - Dh) <= bound * (1 + 1e-9)
    # at 16 bits the fp16 scale (range / 65535) is an fp16 subnormal, so it carries only a few
    # significant bits and the top of the range clamps; the error stays at the percent level
    assert np.linalg.norm(D - Dh) / np.linalg.norm(D) < 1e-2


# --------------------------------------------------------------------------------------------
# Budget and allocation ("Approach": 8/3/2/0 bits, the same size as the 1-bit delta; "Key
# results": 1/16 ratio; "Limitations": 1/32 ratio)
# --------------------------------------------------------------------------------------------
RANK_TABLE = [
    # (d_out, d_in, ratio, widths, expected plan) -- expected ranks worked out by hand:
    # 4096^2 @1/16: B = 4096^2 bits; 8-bit*2 and 3-bit*32 use (16+96)*8192 = 917504 bits;
    #   (16777216 - 917504) / (2*8192) = 968 exactly.
    (4096, 4096, 1 / 16, [(8, 2), (3, 32), (2, None)], [(8, 2), (3, 32), (2, 968)]),
    # 11008x4096: B = 45088768; (16+96)*15104 = 1691648; 43397120 / 30208 = 1436.6 -> 1436
    (11008, 4096, 1 / 16, [(8, 2), (3, 32), (2, None)], [(8, 2), (3, 32), (2, 1436)]),
    (4096, 11008, 1 / 16, [(8, 2), (3, 32), (2, None)], [(8, 2), (3, 32), (2, 1436)]),
    # 13B 5120^2: 26214400 - 112*10240 = 25067520; / 20480 = 1224 exactly
    (5120, 5120, 1 / 16, [(8, 2), (3, 32), (2, None)], [(8, 2), (3, 32), (2, 1224)]),
    # 13824x5120: 70778880 - 112*18944 = 68657152; / 37888 = 1812.1 -> 1812
    (13824, 5120, 1 / 16, [(8, 2), (3, 32), (2, None)], [(8, 2), (3, 32), (2, 1812)]),
    # 1/32 ablation: 8388608 - (8+48)*8192 = 7929856; / 16384 = 484
    (4096, 4096, 1 / 32, [(8, 1), (3, 16), (2, None)], [(8, 1), (3, 16), (2, 484)]),
    # 22544384 - 56*15104 = 21698560; / 30208 = 718.3 -> 718
    (11008, 4096, 1 / 32, [(8, 1), (3, 16), (2, None)], [(8, 1), (3, 16), (2, 718)]),
    # single-precision 3-bit ablation at the 1/16 size: 16777216 / 24576 = 682.7 -> 682
    (4096, 4096, 1 / 16, [(3, None)], [(3, 682)]),
    # 45088768 / 45312 = 995.07 -> 995
    (11008, 4096, 1 / 16, [(3, None)], [(3, 995)]),
    # the budget can never exceed the available rank
    (256, 128, 1.0, [(8, None)], [(8, 128)]),
]


@pytest.mark.parametrize("d_out,d_in,ratio,widths,expected", RANK_TABLE)
def test_rank_table(d_out, d_in, ratio, widths, expected):
    plan = oracle.allocate_ranks(d_out, d_in, ratio, widths)
    assert plan == expected
    if ratio < 1:
        assert oracle.code_bits_used(plan, d_out, d_in) <= oracle.budget_bits(d_out, d_in, ratio)


def test_budget_one_bit_per_parameter_at_one_sixteenth():
    assert oracle.budget_bits(4096, 11008, 1 / 16) == 4096 * 11008


def test_single_linear_plan_bits():
    # 512x512 case, plan (8:2, 3:8, 2:32): (16 + 24 + 64) * 1024 = 106496 code bits
    assert oracle.code_bits_used([(8, 2), (3, 8), (2, 32)], 512, 512) == 106496


# --------------------------------------------------------------------------------------------
# Routing ("Delta-CoMe的应用场景": multi-tenant serving)
# --------------------------------------------------------------------------------------------
def test_route_tokens_matches_stable_sort():
    rng = np.random.default_rng(11)
    for T, n in [(0, 3), (1, 1), (7, 3), (64, 50), (257, 100)]:
        ids = rng.integers(-1, n, size=T).astype(np.int32)
        perm, inv, segs = oracle.route_tokens(ids, n)
        ref = np.argsort(ids, kind="stable")
        assert np.array_equal(perm, ref)
        assert np.array_equal(inv[perm], np.arange(T))
        u, start, cnt = np.unique(ids[ref], return_index=True, return_counts=True)
        expect = [(int(a), int(b), int(c)) for a, b, c in zip(u, start, cnt) if a >= 0]
        assert segs == expect


def test_route_tokens_rejects_bad_ids():
    with pytest.raises(ValueError):
        oracle.route_tokens([0, 3], 3)
    with pytest.raises(ValueError):
        oracle.route_tokens([-2], 3)


# --------------------------------------------------------------------------------------------
# Evaluation (y = W_base x + U_hat (S * (V_hat^T x)))
# --------------------------------------------------------------------------------------------
def _single_case_artefacts(seed=0):
    case = synth.single_linear_case(seed=seed)
    arts = [oracle.compress_delta(oracle.delta_weights(case.w_base, w), case.plan) for w in case.w_ft]
    return case, arts


def test_rank1_closed_form():
    with open(os.path.join(GOLDEN, "rank1_eval.txt")) as f:
        y0 = float([l for l in f if l.startswith("y0")][0].split("=")[1])
    d = 128
    U = np.zeros((d, 1), np.float32); U[0, 0] = 1
    Vt = np.zeros((1, d), np.float32); Vt[0, 1] = 1
    a = oracle.compress_factors(U, np.array([2.0], np.float32), Vt, [(8, 1)])
    x = np.zeros((1, d)); x[0, 1] = 1; x[0, 5] = 3
    y = oracle.delta_linear(np.zeros((d, d)), [a], x, [0])
    assert y[0, 0] == y0
    assert np.all(y[0, 1:] == 0)


def test_segmented_equals_brute_force():
    case, arts = _single_case_artefacts()
    y = oracle.delta_linear(case.w_base, arts, case.x, case.tenant_ids)
    yb = oracle.brute_force_linear(case.w_base, arts, case.x, case.tenant_ids)
    assert np.max(np.abs(y - yb)) <= 1e-12 * np.max(np.abs(yb))


def test_permutation_invariance_and_backbone_only():
    case, arts = _single_case_artefacts()
    rng = np.random.default_rng(9)
    x = rng.standard_normal((9, 512))
    ids = np.array([0, 1, -1, 1, 0, 0, -1, 1, 1], dtype=np.int32)
    y = oracle.delta_linear(case.w_base, arts, x, ids)
    p = rng.permutation(9)
    yp = oracle.delta_linear(case.w_base, arts, x[p], ids[p])
    assert np.array_equal(yp, y[p])
    base = x @ case.w_base.astype(np.float64).T
    assert np.array_equal(y[ids == -1], base[ids == -1])
    # one token alone gives the same row as inside the batch
    y1 = oracle.delta_linear(case.w_base, arts, x[3:4], ids[3:4])
    assert np.allclose(y1[0], y[3], rtol=0, atol=1e-14)


def test_zero_bit_ranks_contribute_nothing():
    case = synth.single_linear_case(seed=0)
    D = oracle.delta_weights(case.w_base, case.w_ft[0])
    U, s, Vt = oracle.svd_factors(D)
    f32 = lambda a: a.astype(np.float32)
    a1 = oracle.compress_factors(f32(U), f32(s), f32(Vt), [(8, 2), (3, 8), (2, 32)])
    a2 = oracle.compress_factors(f32(U), f32(s), f32(Vt), [(8, 2), (3, 8), (2, 32), (0, 100)])
    ids = np.zeros(4, np.int32)
    assert np.array_equal(oracle.delta_linear(case.w_base, [a1], case.x, ids),
                          oracle.delta_linear(case.w_base, [a2], case.x, ids))
    assert a2.rank == 42 and a2.u_codes.shape == (42, 512)


def test_single_tenant_batch_equals_one_matrix():
    case, arts = _single_case_artefacts()
    ids = np.ones(5, np.int32)
    x = np.random.default_rng(2).standard_normal((5, 512))
    Uh, S, Vt = oracle.dequantized_factors(arts[1])
    M = case.w_base.astype(np.float64) + (Uh * S) @ Vt
    y = oracle.delta_linear(case.w_base, arts, x, ids)
    assert np.max(np.abs(y - x @ M.T)) <= 1e-12 * np.max(np.abs(y))


def test_delta_only_rows_subset():
    case, arts = _single_case_artefacts()
    rows = np.array([0, 5, 127, 128, 511])
    full = oracle.delta_only(arts, case.x, case.tenant_ids)
    sub = oracle.delta_only(arts, case.x, case.tenant_ids, rows=rows)
    assert np.allclose(sub, full[:, rows], rtol=0, atol=1e-15)


def test_activation_error_small_and_ordered():
    # more bits / more ranks -> smaller activation approximation error ("Experimental setup"
    # lists activation approximation error; "Approach": more bits for larger singular values)
    case = synth.single_linear_case(seed=0)
    D = oracle.delta_weights(case.w_base, case.w_ft[0])
    U, s, Vt = oracle.svd_factors(D)
    f32 = lambda a: a.astype(np.float32)
    x = np.random.default_rng(4).standard_normal((16, 512))
    e_mixed = oracle.activation_error(D, oracle.compress_factors(f32(U), f32(s), f32(Vt), [(8, 2), (3, 8), (2, 32)]), x)
    e_more = oracle.activation_error(D, oracle.compress_factors(f32(U), f32(s), f32(Vt), [(8, 64), (3, 64)]), x)
    e_full = oracle.activation_error(D, oracle.compress_factors(f32(U), f32(s), f32(Vt), [(16, 512)]), x)
    assert e_full < e_more < e_mixed < 1.0
    assert e_full < 1e-2   # 16-bit grids have fp16-subnormal scales (see the test above)


def test_activation_error_equals_frobenius_error_of_the_explicit_matrix():
    # With X = I the activation error is ||Delta - Delta_hat||_F / ||Delta||_F, Delta_hat formed
    # explicitly as sum_i S_i u_hat_i v_hat_i^T; an orthogonal X or a scaled X leaves it unchanged
    # (the Frobenius norm is invariant under rotations, the ratio under scaling).  The shape is
    # not square, so a transposed evaluation fails.
    rng = np.random.default_rng(31)
    d_out, d_in = 256, 384
    Q1, _ = np.linalg.qr(rng.standard_normal((d_out, d_out)))
    Q2, _ = np.linalg.qr(rng.standard_normal((d_in, d_out)))
    D = Q1 @ np.diag(0.05 / np.arange(1, d_out + 1)) @ Q2.T
    a = oracle.compress_delta(D, [(8, 2), (3, 16), (2, 48)])
    Uh, S, Vt = oracle.dequantized_factors(a)
    M = np.zeros((d_out, d_in))
    for i in range(S.shape[0]):
        for o in range(d_out):
            M[o] += S[i] * Uh[o, i] * Vt[i]
    want = np.linalg.norm(D - M) / np.linalg.norm(D)
    assert 1e-3 < want < 1.0
    assert abs(oracle.activation_error(D, a, np.eye(d_in)) - want) <= 1e-12 * want
    R, _ = np.linalg.qr(rng.standard_normal((d_in, d_in)))
    assert abs(oracle.activation_error(D, a, R) - want) <= 1e-10 * want
    assert abs(oracle.activation_error(D, a, 3.0 * R) - want) <= 1e-10 * want


def test_long_tail_mixed_precision_beats_single_precision_same_size():
    # "Measured effects" table: adding 8- and 2-bit groups to a single-precision 3-bit setting of
    # the same size helped.  On a long-tail spectrum the activation error must order the same way.
    rng = np.random.default_rng(21)
    d = 512
    q1 = synth.random_orthonormal(rng, d, d)
    q2 = synth.random_orthonormal(rng, d, d)
    s = 0.02 * math.sqrt(d) * np.arange(1, d + 1) ** -0.8
    D = (q1 * s) @ q2.T
    U, sig, Vt = oracle.svd_factors(D)
    f32 = lambda a: a.astype(np.float32)
    mixed = oracle.allocate_ranks(d, d, 1 / 16, [(8, 2), (3, 32), (2, None)])
    single3 = oracle.allocate_ranks(d, d, 1 / 16, [(3, None)])
    x = rng.standard_normal((32, d))
    e_mixed = oracle.activation_error(D, oracle.compress_factors(f32(U), f32(sig), f32(Vt), mixed), x)
    e_three = oracle.activation_error(D, oracle.compress_factors(f32(U), f32(sig), f32(Vt), single3), x)
    assert e_mixed < e_three


# --------------------------------------------------------------------------------------------
# Input generator (not the method): bf16 rounding and the counter-based stream
# --------------------------------------------------------------------------------------------
def test_bf16_round_ties_to_even():
    bits, vals = synth.bf16_round(np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5], np.float32))
    assert list(vals) == [1.0, 1.0 + 2 ** -6, -2.5]


def test_splitmix64_reference_values():
    # SplitMix64 with state starting at 0: published first outputs of the generator
    # (seed 0 -> 0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F)
    g = np.uint64(0x9E3779B97F4A7C15)
    with np.errstate(over="ignore"):
        out = synth.mix64(np.arange(1, 4, dtype=np.uint64) * g)
    assert [int(v) for v in out] == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


def test_stream_normal_moments_and_slices():
    x = synth.stream_normal(3, 17, 0, 200000, 2.0)
    assert abs(x.mean()) < 0.02 and abs(x.std() - 2.0) < 0.02
    assert np.array_equal(synth.stream_normal(3, 17, 1000, 50, 2.0), x[1000:1050])
