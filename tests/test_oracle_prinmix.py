"""Pins of the PrinMix oracle (oracle/prinmix.py) and CPU parity of the library's host PrinMix
routines against it.

Page: "Enhancing Delta Compression in LLMs via SVD-based Quantization Error Minimization", sections
2.1 (eq. 5), 2.2 (0/1 ILP), 2.3 (reconstruction-target correction), 2.4 (order of the steps).
"""
import numpy as np
import pytest

import oracle
from oracle import prinmix as pm
import tenant_mixed_precision_b200 as dc


def _case(seed=0, d_out=256, d_in=384, r=24, n=48):
    rng = np.random.default_rng(seed)
    U, _ = np.linalg.qr(rng.standard_normal((d_out, r)))
    V, _ = np.linalg.qr(rng.standard_normal((d_in, r)))
    S = 0.5 * np.arange(1, r + 1) ** -0.8
    X = rng.standard_normal((n, d_in))
    return U, S, V.T.copy(), X


# ---------------------------------------------------------------------------------------- oracle pins
def test_eq5_is_exact_for_one_row_with_orthonormal_U():
    # with orthonormal columns of U, quantising row i alone changes U diag(S) V X^T by exactly
    # S_i^2 |dV_i X^T|^2 in squared Frobenius norm (eq. 5 without its approximation)
    U, S, Vt, X = _case()
    sc = pm.error_scores(Vt, S, X)
    full = (U * S) @ Vt @ X.T
    for i in (0, 5, 23):
        for j, b in enumerate(pm.WIDTHS):
            V2 = Vt.copy()
            V2[i] = pm.quantised_row(Vt[i], b)
            err = np.linalg.norm(full - (U * S) @ V2 @ X.T) ** 2
            assert abs(err - sc[i, j]) <= 1e-9 * max(err, 1e-300), (i, b)


def test_scores_order_and_drop_term():
    U, S, Vt, X = _case(1)
    sc = pm.error_scores(Vt, S, X)
    # 0 bits drops the row: the whole row's output; more bits never hurt
    assert np.allclose(sc[:, 0], S ** 2 * np.sum((X @ Vt.T) ** 2, axis=0), rtol=1e-12)
    assert np.all(sc[:, 0] >= sc[:, 1]) and np.all(sc[:, 1] >= sc[:, 2]) and np.all(sc[:, 2] >= sc[:, 3])


@pytest.mark.parametrize("max_kinds", [1, 2, 3])
def test_ilp_equals_brute_force(max_kinds):
    rng = np.random.default_rng(10 + max_kinds)
    for trial in range(4):
        r = 6
        sc = np.sort(rng.exponential(size=(r, 4)), axis=1)[:, ::-1] * rng.uniform(0.1, 3, size=(r, 1))
        d_out, d_in = 128, 128
        ratio = rng.uniform(0.01, 0.05)
        w_i, e_i = pm.allocate_ilp(sc, pm.WIDTHS, d_out, d_in, ratio, max_kinds)
        w_b, e_b = pm.allocate_brute_force(sc, pm.WIDTHS, d_out, d_in, ratio, max_kinds)
        assert abs(e_i - e_b) <= 1e-9 * max(1.0, e_b)
        cap = pm.budget_units(d_out, d_in, ratio)
        assert int(np.sum(w_i)) <= cap and len({b for b in w_i if b}) <= max_kinds


def test_ilp_never_worse_than_the_greedy_plan():
    # the greedy 8/3/2 plan is one feasible point of the ILP with 3 kinds
    U, S, Vt, X = _case(2, d_out=512, d_in=512, r=96, n=64)
    sc = pm.error_scores(Vt, S, X)
    ratio = 1 / 16 * 0.25
    greedy = oracle.allocate_ranks(512, 512, ratio, [(8, 2), (3, 8), (2, None)])
    gw = np.zeros(96, np.int64)
    k = 0
    for b, n in greedy:
        gw[k:k + n] = b
        k += n
    col = {b: j for j, b in enumerate(pm.WIDTHS)}
    e_greedy = sum(sc[i, col[int(gw[i])]] for i in range(96))
    _, e_ilp = pm.allocate_ilp(sc, pm.WIDTHS, 512, 512, ratio, 3)
    assert e_ilp <= e_greedy * (1 + 1e-12)


def test_rtc_normal_equations_and_improvement():
    U, S, Vt, X = _case(3)
    Vh = np.stack([pm.quantised_row(v, 2) for v in Vt])
    Ut = pm.rtc(U, S, Vt, Vh, X)
    A = (Vh @ X.T) * S[:, None]
    B = (Vt @ X.T) * S[:, None]
    grad = (Ut @ A - U @ B) @ A.T
    assert np.abs(grad).max() <= 1e-9 * np.abs(U @ B @ A.T).max()
    obj = lambda W: np.linalg.norm(U @ B - W @ A)
    assert obj(Ut) <= obj(U) * (1 + 1e-12)
    # exact V_hat: nothing to correct
    assert np.allclose(pm.rtc(U, S, Vt, Vt, X), U, atol=1e-10)


def test_compress_prinmix_plan_and_budget():
    U, S, Vt, X = _case(4, d_out=256, d_in=256, r=64, n=96)
    art, w, perm = pm.compress_prinmix(U, S, Vt, X, ratio=1 / 64, max_kinds=3)
    assert [b for b, _ in art.plan] == sorted({int(b) for b in w if b}, reverse=True)
    assert sum(n for _, n in art.plan) == len(perm) == int(np.sum(w > 0))
    assert oracle.code_bits_used(art.plan, 256, 256) <= 1 / 64 * 16 * 256 * 256
    assert all(w[perm[i]] >= w[perm[i + 1]] for i in range(len(perm) - 1))


# ------------------------------------------------------------------ library host routines vs oracle
def test_library_scores_match_oracle():
    U, S, Vt, X = _case(5)
    got = dc.dc_prinmix_scores(Vt, S, X)
    want = pm.error_scores(Vt.astype(np.float32), S.astype(np.float32), X.astype(np.float32))
    assert np.allclose(got, want, rtol=1e-9, atol=0)


@pytest.mark.parametrize("max_kinds", [1, 2, 3])
def test_library_allocation_is_optimal(max_kinds):
    U, S, Vt, X = _case(6, d_out=512, d_in=512, r=128, n=64)
    sc = pm.error_scores(Vt, S, X)
    for ratio in (1 / 64, 1 / 32):
        w, obj = dc.dc_prinmix_allocate(sc, pm.WIDTHS, 512, 512, ratio, max_kinds)
        _, e_ilp = pm.allocate_ilp(sc, pm.WIDTHS, 512, 512, ratio, max_kinds)
        col = {b: j for j, b in enumerate(pm.WIDTHS)}
        e_w = sum(sc[i, col[int(w[i])]] for i in range(len(w)))
        assert abs(obj - e_w) <= 1e-9 * e_w
        assert abs(obj - e_ilp) <= 1e-9 * max(e_ilp, 1e-300), (obj, e_ilp)
        assert int(np.sum(w)) <= pm.budget_units(512, 512, ratio) and len({b for b in w if b}) <= max_kinds


def test_library_rtc_matches_oracle():
    U, S, Vt, X = _case(7)
    Vh = np.stack([pm.quantised_row(v, 3) for v in Vt.astype(np.float32)])
    got = dc.dc_prinmix_rtc(U, S, Vt, Vh, X)
    want = pm.rtc(U.astype(np.float32), S.astype(np.float32), Vt.astype(np.float32), Vh.astype(np.float32),
                  X.astype(np.float32))
    assert np.abs(got - want).max() <= 1e-5 * np.abs(want).max()


def test_library_compress_matches_oracle():
    U, S, Vt, X = _case(8, d_out=256, d_in=384, r=48, n=96)
    desc, perm, Uo, So, Vo, obj = dc.dc_prinmix_compress(U, S, Vt, X, ratio=1 / 64, max_kinds=3)
    art, w, operm = pm.compress_prinmix(U.astype(np.float32), S.astype(np.float32), Vt.astype(np.float32),
                                        X.astype(np.float32), ratio=1 / 64, max_kinds=3)
    plan = [(desc.bits[i], desc.rank[i]) for i in range(desc.n_bands)]
    assert plan == art.plan
    assert list(perm[: len(operm)]) == list(operm) and np.all(perm[len(operm):] == -1)
    assert np.array_equal(So, S.astype(np.float32)[operm])
    Uh, _, _ = oracle.dequantized_factors(art)
    # the refit U agrees with the oracle's to fp32 rounding (its quantised codes may differ only
    # where a value sits on a rounding boundary)
    Uw = pm.rtc(U[:, operm].astype(np.float32), S[operm].astype(np.float32), Vt[operm].astype(np.float32),
                np.stack([pm.quantised_row(Vt[i].astype(np.float32), int(w[i])) for i in operm]), X.astype(np.float32))
    assert np.abs(Uo - Uw).max() <= 1e-5 * np.abs(Uw).max()
