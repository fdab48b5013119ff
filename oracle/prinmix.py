"""fp64 reference of the PrinMix allocation variants (offline steps before the serving path).

TEST INFRASTRUCTURE ONLY (see the package docstring): the product never imports this file.

Source: [P4] "Enhancing Delta Compression in LLMs via SVD-based Quantization Error Minimization"
(gist.science explanation of PrinMix, a follow-up to Delta-CoMe with the same factorisation
W = U Sigma V):

* section 2.1, eq. 5: quantising row i of V changes the output on calibration activations X by
  approximately Sigma_ii^2 * dV_i X X^T dV_i^T ("scaling" term times "difference" term);
* section 2.2: the bit allocation is a 0/1 integer linear program -- minimise the summed error
  subject to a bit budget, one width per row (one-hot), widths from a candidate set, and at most a
  given number of distinct widths; the page solves it with CVXPY and SCIP;
* section 2.3: reconstruction-target correction (RTC): before U is quantised it is replaced by the
  least-squares solution of min |U Sigma V X - U~ Sigma V_hat X|_F^2, V_hat the quantised V;
* section 2.4: SVD, error terms per width, ILP, RTC, quantise.

Readings (listed in the design doc as well):

R-P1  dV_i for width b is v_i minus its round-to-nearest image at b bits under the serving rule
      (reading R1 of delta_come.py, groups of 128 along d_in); for 0 bits dV_i = v_i (the row is
      dropped).
R-P2  Widths come from {0, 2, 3, 8} (what the serving layout stores); 0 is always allowed; a width
      b costs b * (d_out + d_in) code bits per rank; the budget is ratio * 16 * d_out * d_in code
      bits (reading R2); "at most K distinct widths" counts nonzero widths.
R-P3  RTC refits the kept ranks only: the target is U_k Sigma_k V_k X over the ranks with a nonzero
      width, and U~ replaces U_k.
R-P4  The kept ranks are grouped into bands by width, widest first (8, 3, 2), singular-value order
      inside a band, so that the serving layout's bands hold them; the product is unchanged by
      that reordering.

Parity: eq. 5 is pinned by its exact form for one row with orthonormal U; the ILP by brute-force
enumeration on small instances; RTC by the normal equations (zero gradient) and by never doing
worse than no correction (tests/test_oracle_prinmix.py).
"""
from __future__ import annotations

import itertools

import numpy as np

from .delta_come import compress_factors, rtn_quantize_vector, dequantize_vector

WIDTHS = (0, 2, 3, 8)


def quantised_row(v: np.ndarray, bits: int) -> np.ndarray:
    """RTN image of one row of V at `bits` (zeros for 0 bits), fp64."""
    v = np.asarray(v, dtype=np.float64)
    if bits == 0:
        return np.zeros_like(v)
    return dequantize_vector(rtn_quantize_vector(v, bits))


def error_scores(Vt: np.ndarray, S: np.ndarray, X: np.ndarray, widths=WIDTHS) -> np.ndarray:
    """Eq. 5 of [P4] 2.1 for every row i and width b: S_i^2 * |dV_i(b) X^T|^2.

    Vt: [r, d_in] rows v_i; S: [r]; X: [n, d_in] calibration tokens (rows).  Returns [r, len(widths)].
    """
    Vt = np.asarray(Vt, dtype=np.float64)
    X = np.asarray(X, dtype=np.float64)
    S = np.asarray(S, dtype=np.float64)
    out = np.zeros((Vt.shape[0], len(widths)))
    for i in range(Vt.shape[0]):
        for j, b in enumerate(widths):
            dv = Vt[i] - quantised_row(Vt[i], b)
            p = X @ dv
            out[i, j] = S[i] ** 2 * float(p @ p)
    return out


def budget_units(d_out: int, d_in: int, ratio: float) -> int:
    """The bit budget ratio * 16 * d_out * d_in in units of d_out + d_in bits (one bit per rank)."""
    return int(np.floor(ratio * 16.0 * d_out * d_in / (d_out + d_in) + 1e-9))


def allocate_ilp(scores: np.ndarray, widths, d_out: int, d_in: int, ratio: float, max_kinds: int):
    """The 0/1 ILP of [P4] 2.2, solved with a library MILP solver (scipy's HiGHS), one binary
    s_ib per (row, width) and one binary z_b per nonzero width:

        min  sum_ib e_ib s_ib
        s.t. sum_b s_ib = 1                       (one-hot)
             sum_ib b s_ib <= budget units        (bit budget)
             s_ib <= z_b,  sum_b z_b <= max_kinds (at most max_kinds distinct nonzero widths)

    Returns (widths per row, objective)."""
    from scipy.optimize import Bounds, LinearConstraint, milp

    scores = np.asarray(scores, dtype=np.float64)
    r, m = scores.shape
    widths = list(widths)
    nzb = [j for j, b in enumerate(widths) if b != 0]
    nv = r * m + len(nzb)
    c = np.concatenate([scores.reshape(-1), np.zeros(len(nzb))])
    rows, lo, hi = [], [], []
    for i in range(r):  # one-hot
        a = np.zeros(nv)
        a[i * m:(i + 1) * m] = 1.0
        rows.append(a), lo.append(1.0), hi.append(1.0)
    a = np.zeros(nv)  # budget
    for i in range(r):
        for j, b in enumerate(widths):
            a[i * m + j] = b
    rows.append(a), lo.append(-np.inf), hi.append(float(budget_units(d_out, d_in, ratio)))
    for k, j in enumerate(nzb):  # s_ij <= z_j
        for i in range(r):
            a = np.zeros(nv)
            a[i * m + j] = 1.0
            a[r * m + k] = -1.0
            rows.append(a), lo.append(-np.inf), hi.append(0.0)
    a = np.zeros(nv)
    a[r * m:] = 1.0
    rows.append(a), lo.append(-np.inf), hi.append(float(max_kinds))
    res = milp(c, constraints=LinearConstraint(np.array(rows), lo, hi), integrality=np.ones(nv),
               bounds=Bounds(0, 1), options={"mip_rel_gap": 0.0})
    if not res.success:
        raise RuntimeError(f"ILP not solved: {res.message}")
    s = np.round(res.x[: r * m]).reshape(r, m)
    w = np.array([widths[int(np.argmax(s[i]))] for i in range(r)], dtype=np.int64)
    return w, float(np.sum(scores * s))


def allocate_brute_force(scores, widths, d_out: int, d_in: int, ratio: float, max_kinds: int):
    """Every assignment of widths to rows (tiny instances only); the feasible one of least error."""
    scores = np.asarray(scores, dtype=np.float64)
    r, m = scores.shape
    cap = budget_units(d_out, d_in, ratio)
    best, best_w = np.inf, None
    for combo in itertools.product(range(m), repeat=r):
        ws = [widths[j] for j in combo]
        if sum(ws) > cap or len({b for b in ws if b}) > max_kinds:
            continue
        e = sum(scores[i, j] for i, j in enumerate(combo))
        if e < best:
            best, best_w = e, np.array(ws, dtype=np.int64)
    return best_w, float(best)


def rtc(U: np.ndarray, S: np.ndarray, Vt: np.ndarray, Vt_hat: np.ndarray, X: np.ndarray) -> np.ndarray:
    """[P4] 2.3: U~ = argmin |U diag(S) V X^T - U~ diag(S) V_hat X^T|_F, by a library least-squares
    solve (each row of U~ is an independent least-squares problem).  U: [d_out, k] columns u_i."""
    U = np.asarray(U, dtype=np.float64)
    S = np.asarray(S, dtype=np.float64)
    X = np.asarray(X, dtype=np.float64)
    B = (np.asarray(Vt, dtype=np.float64) @ X.T) * S[:, None]      # [k, n]
    A = (np.asarray(Vt_hat, dtype=np.float64) @ X.T) * S[:, None]  # [k, n]
    target = U @ B                                                # [d_out, n]
    sol, *_ = np.linalg.lstsq(A.T, target.T, rcond=None)          # A^T U~^T = target^T
    return sol.T


def compress_prinmix(U, S, Vt, X, ratio: float, max_kinds: int, widths=WIDTHS, use_rtc: bool = True,
                     d_out: int | None = None, d_in: int | None = None):
    """[P4] 2.4 in order: error terms per width, ILP, bands by width (R-P4), RTC, quantise.

    U: [d_out, r] (columns u_i), S: [r], Vt: [r, d_in] -- the candidate ranks from the SVD.
    Returns (artefact, widths per candidate rank, permutation: source rank of each kept rank)."""
    U = np.asarray(U, dtype=np.float64)
    Vt = np.asarray(Vt, dtype=np.float64)
    S = np.asarray(S, dtype=np.float64)
    d_out = U.shape[0] if d_out is None else d_out
    d_in = Vt.shape[1] if d_in is None else d_in
    sc = error_scores(Vt, S, X, widths)
    w, _ = allocate_ilp(sc, widths, d_out, d_in, ratio, max_kinds)
    perm = [i for b in (8, 3, 2) for i in range(len(w)) if w[i] == b]
    plan = [(b, int(np.sum(w == b))) for b in (8, 3, 2) if np.sum(w == b) > 0]
    Uk, Sk, Vk = U[:, perm], S[perm], Vt[perm]
    if use_rtc and perm:
        bits = np.array([w[i] for i in perm])
        Vh = np.stack([quantised_row(Vk[i], int(bits[i])) for i in range(len(perm))])
        Uk = rtc(Uk, Sk, Vk, Vh, X)
    art = compress_factors(Uk.astype(np.float32), Sk.astype(np.float32), Vk.astype(np.float32), plan)
    return art, w, np.array(perm, dtype=np.int64)
