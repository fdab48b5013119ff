"""fp64 reference of Delta-CoMe mixed-precision delta compression and multi-tenant evaluation.

TEST INFRASTRUCTURE ONLY (see the package docstring): the product never imports this file.

Notation follows the pages.  A fine-tuned linear W_ft (d_out x d_in) is the backbone W_base plus
a delta Delta = W_ft - W_base.  Its SVD is Delta = U diag(sigma) V^T; u_i is column i of U
(length d_out) and v_i^T is row i of V^T (length d_in), in descending sigma.  Each rank i is
stored at a bit width b_i in {8, 3, 2, 0}; 0-bit ranks are dropped.  A kept rank stores its two
vectors quantised by round-to-nearest in groups of 128 consecutive elements (one fp16 scale and
one fp16 zero point per group) and its singular value as fp32 S_i.  Serving computes, for a
token x with tenant tau,

    y = W_base x + U_hat_tau (S_tau * (V_hat_tau^T x)).

Readings of points the pages leave open (each is restated where it is used):

R1  RTN grid: asymmetric min/max with 0 forced into the range, qmax = 2**b - 1,
    scale = fp16_rne((hi - lo) / qmax) (1 if that is 0), zero = clamp(rint(-lo / scale)),
    code = clamp(rint(v / scale) + zero); rint is round-half-to-even in fp64 and uses the
    fp16-rounded scale.  Group size 128 along each vector's length.
R2  Budget: ratio * 16 * d_out * d_in code bits (1/16 -> one bit per delta parameter, the size
    of a 1-bit delta); scales, zeros and S are not charged to it.
R3  Greedy allocation: the bit groups are filled in descending-sigma order from a width plan
    such as [(8, 2), (3, 32), (2, None)], where None means "as many as the budget still allows".
R4  SVD sign: each pair (u_i, v_i) is flipped so that the entry of v_i of largest magnitude is
    positive (lowest index on ties).
R5  Tenant id -1 means "backbone only" for that token.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np

GROUP = 128


# ------------------------------------------------------------------------------------------
# Step 1: the delta.  [P1] "Delta-CoMe的技术原理" (low-rank decomposition of the parameter
# delta); [P2] "Approach" (fine-tuned minus backbone weights).  Parity: pinned (exact fp64).
# ------------------------------------------------------------------------------------------
def delta_weights(w_base: np.ndarray, w_ft: np.ndarray) -> np.ndarray:
    return np.asarray(w_ft, dtype=np.float64) - np.asarray(w_base, dtype=np.float64)


# ------------------------------------------------------------------------------------------
# Step 2: SVD with the sign convention R4.  [P1] "Delta-CoMe的技术原理" (SVD of the delta);
# [P4] 2.1 (W = U Sigma V).  The routine is LAPACK (numpy.linalg.svd).  Parity: pinned by
# reconstruction, orthonormality and recovery of a constructed spectrum.
# ------------------------------------------------------------------------------------------
def svd_factors(delta: np.ndarray):
    """Return (U [d_out, m], sigma [m], Vt [m, d_in]) in descending sigma, signs fixed (R4)."""
    U, s, Vt = np.linalg.svd(np.asarray(delta, dtype=np.float64), full_matrices=False)
    U = U.copy()
    Vt = Vt.copy()
    for i in range(s.shape[0]):
        j = int(np.argmax(np.abs(Vt[i])))   # first index of the largest magnitude
        if Vt[i, j] < 0:
            Vt[i] *= -1.0
            U[:, i] *= -1.0
    return U, s, Vt


def eckart_young_tail(sigma: np.ndarray, k: int) -> float:
    """Frobenius error of the best rank-k approximation: sqrt(sum_{i>k} sigma_i^2)."""
    s = np.asarray(sigma, dtype=np.float64)
    return float(math.sqrt(float(np.sum(s[k:] ** 2))))


# ------------------------------------------------------------------------------------------
# Budget and greedy allocation.  [P2] "Approach" (8/3/2-bit groups for successive singular
# vectors, the smallest dropped as 0-bit, the same size as the 1-bit delta baseline) and
# "Key results"/"Limitations" (a preliminary greedy search chose the allocation; 1/16 and 1/32
# ratios).  Readings R2, R3.  Parity: pinned by the closed-form rank table.
# ------------------------------------------------------------------------------------------
def budget_bits(d_out: int, d_in: int, ratio: float) -> float:
    return ratio * 16.0 * d_out * d_in


def code_bits_used(plan, d_out: int, d_in: int) -> int:
    return int(sum(b * r * (d_out + d_in) for b, r in plan))


def allocate_ranks(d_out: int, d_in: int, ratio: float, widths) -> list[tuple[int, int]]:
    """Fill bit groups in descending-sigma order; returns [(bits, rank), ...] (0-bit omitted)."""
    cap = min(d_out, d_in)
    budget = budget_bits(d_out, d_in, ratio)
    per_rank = d_out + d_in
    used = 0
    taken = 0
    plan = []
    for bits, count in widths:
        if bits <= 0:
            continue
        if count is None:
            count = int(math.floor((budget - used) / (bits * per_rank)))
        count = max(0, min(int(count), cap - taken))
        plan.append((int(bits), count))
        used += bits * count * per_rank
        taken += count
    return plan


# ------------------------------------------------------------------------------------------
# RTN quantisation, reading R1.  [P1] "Delta-CoMe的技术原理" (mixed-precision quantisation of
# the singular vectors: larger singular values get more bits); [P2] "Approach".  The group
# size 128, the fp16 scale/zero and round-to-nearest are the serving format this build fixes.
# Parity: pinned by hand-derived codes (tests/golden/rtn_groups.txt), tie cases, the
# |v - v_hat| <= scale/2 bound and brute-force nearest-grid-point search.
# ------------------------------------------------------------------------------------------
def _fp16(x: float) -> float:
    return float(np.float16(x))


def rtn_quantize_group(g: np.ndarray, bits: int):
    """Quantise one group.  Returns (codes int64, scale float (an fp16 value), zero float)."""
    g = np.asarray(g, dtype=np.float64)
    if not np.all(np.isfinite(g)):
        raise ValueError("non-finite value in a quantisation group")
    qmax = (1 << bits) - 1
    lo = min(0.0, float(g.min()))
    hi = max(0.0, float(g.max()))
    scale = _fp16((hi - lo) / qmax)
    if not math.isfinite(scale):
        raise ValueError("group range overflows the fp16 scale")
    if scale == 0.0:
        scale = 1.0
    zero = float(min(max(np.rint(-lo / scale), 0.0), float(qmax)))
    codes = np.clip(np.rint(g / scale) + zero, 0.0, float(qmax)).astype(np.int64)
    return codes, scale, zero


@dataclass
class QuantVector:
    codes: np.ndarray    # int64 [n]
    scales: np.ndarray   # float64 [n_groups] (fp16 values)
    zeros: np.ndarray    # float64 [n_groups] (integers)
    bits: int


def rtn_quantize_vector(v: np.ndarray, bits: int, group: int = GROUP) -> QuantVector:
    """Quantise a vector group by group (plain loop over rtn_quantize_group)."""
    v = np.asarray(v, dtype=np.float64)
    n = v.shape[0]
    codes = np.empty(n, dtype=np.int64)
    ng = (n + group - 1) // group
    scales = np.empty(ng)
    zeros = np.empty(ng)
    for gi in range(ng):
        sl = slice(gi * group, min(n, (gi + 1) * group))
        c, s, z = rtn_quantize_group(v[sl], bits)
        codes[sl] = c
        scales[gi] = s
        zeros[gi] = z
    return QuantVector(codes, scales, zeros, bits)


def _rtn_quantize_rows(M: np.ndarray, bits: int, group: int = GROUP):
    """Same rule as rtn_quantize_group, applied to every group of every row of M at once.

    M is [n_vec, n] with n a multiple of ``group``.  Returns codes int64 [n_vec, n], scales and
    zeros float64 [n_vec, n // group].
    """
    M = np.asarray(M, dtype=np.float64)
    nv, n = M.shape
    if n % group:
        out = [rtn_quantize_vector(M[i], bits, group) for i in range(nv)]
        return (np.stack([o.codes for o in out]), np.stack([o.scales for o in out]),
                np.stack([o.zeros for o in out]))
    if not np.all(np.isfinite(M)):
        raise ValueError("non-finite value in a quantisation group")
    G = M.reshape(nv, n // group, group)
    qmax = float((1 << bits) - 1)
    lo = np.minimum(0.0, G.min(axis=2))
    hi = np.maximum(0.0, G.max(axis=2))
    scale = ((hi - lo) / qmax).astype(np.float16).astype(np.float64)
    if not np.all(np.isfinite(scale)):
        raise ValueError("group range overflows the fp16 scale")
    scale[scale == 0.0] = 1.0
    zero = np.clip(np.rint(-lo / scale), 0.0, qmax)
    codes = np.clip(np.rint(G / scale[:, :, None]) + zero[:, :, None], 0.0, qmax)
    return codes.reshape(nv, n).astype(np.int64), scale, zero


def dequantize_vector(q: QuantVector, group: int = GROUP) -> np.ndarray:
    """v_hat = (code - zero) * scale, in fp64."""
    n = q.codes.shape[0]
    gidx = np.arange(n) // group
    return (q.codes.astype(np.float64) - q.zeros[gidx]) * q.scales[gidx]


# ------------------------------------------------------------------------------------------
# The compressed artefact of one tenant's linear.
# ------------------------------------------------------------------------------------------
@dataclass
class Artefact:
    d_out: int
    d_in: int
    plan: list            # [(bits, rank), ...] in descending-sigma order; 0-bit ranks omitted
    S: np.ndarray         # float32 [r]
    u_codes: np.ndarray   # int64 [r, d_out]   (row i = codes of u_i)
    u_scales: np.ndarray  # float64 [r, d_out // 128]
    u_zeros: np.ndarray
    v_codes: np.ndarray   # int64 [r, d_in]    (row i = codes of v_i)
    v_scales: np.ndarray  # float64 [r, d_in // 128]
    v_zeros: np.ndarray

    @property
    def rank(self) -> int:
        return int(sum(r for _, r in self.plan))

    def bits_per_rank(self) -> np.ndarray:
        return np.concatenate([np.full(r, b, dtype=np.int64) for b, r in self.plan]) if self.plan else \
            np.zeros(0, dtype=np.int64)


def compress_factors(U: np.ndarray, S: np.ndarray, Vt: np.ndarray, plan) -> Artefact:
    """Quantise given SVD factors under a plan [(bits, rank), ...] (ranks past the plan dropped).

    [P2] "Approach": bit groups for successive singular vectors, smallest ranks 0-bit.
    [P4] 2.1/2.3: V is quantised row-wise, and V before U (the order is immaterial for RTN).
    S is stored as fp32.  Parity: pinned (reconstruction, 0-bit invariance, bounds).
    """
    U = np.asarray(U, dtype=np.float64)
    Vt = np.asarray(Vt, dtype=np.float64)
    d_out, d_in = U.shape[0], Vt.shape[1]
    plan = [(int(b), int(r)) for b, r in plan if int(b) > 0 and int(r) > 0]
    r_tot = sum(r for _, r in plan)
    if r_tot > min(U.shape[1], Vt.shape[0]):
        raise ValueError("plan asks for more ranks than the factors hold")
    ng_o = (d_out + GROUP - 1) // GROUP
    ng_i = (d_in + GROUP - 1) // GROUP
    uc = np.zeros((r_tot, d_out), dtype=np.int64)
    us = np.zeros((r_tot, ng_o))
    uz = np.zeros((r_tot, ng_o))
    vc = np.zeros((r_tot, d_in), dtype=np.int64)
    vs = np.zeros((r_tot, ng_i))
    vz = np.zeros((r_tot, ng_i))
    start = 0
    for bits, r in plan:
        sl = slice(start, start + r)
        vc[sl], vs[sl], vz[sl] = _rtn_quantize_rows(Vt[sl], bits)
        uc[sl], us[sl], uz[sl] = _rtn_quantize_rows(U[:, sl].T, bits)
        start += r
    S32 = np.asarray(S[:r_tot], dtype=np.float32).copy()
    return Artefact(d_out, d_in, plan, S32, uc, us, uz, vc, vs, vz)


def compress_delta(delta: np.ndarray, plan) -> Artefact:
    """SVD the delta (R4 signs), then quantise the plan's ranks.  Factors pass through fp32, the
    precision in which the serving library receives them."""
    U, s, Vt = svd_factors(delta)
    return compress_factors(U.astype(np.float32), s.astype(np.float32), Vt.astype(np.float32), plan)


def _dequant_rows(codes, scales, zeros, group=GROUP):
    n = codes.shape[1]
    gidx = np.arange(n) // group
    return (codes.astype(np.float64) - zeros[:, gidx]) * scales[:, gidx]


def dequantized_factors(a: Artefact, u_rows=None):
    """(U_hat [d_out or len(u_rows), r], S fp64 [r], Vt_hat [r, d_in]) in fp64."""
    Vt = _dequant_rows(a.v_codes, a.v_scales, a.v_zeros)
    if u_rows is None:
        Uh = _dequant_rows(a.u_codes, a.u_scales, a.u_zeros).T
    else:
        rows = np.asarray(u_rows)
        Uh = ((a.u_codes[:, rows].astype(np.float64) - a.u_zeros[:, rows // GROUP])
              * a.u_scales[:, rows // GROUP]).T
    return Uh, a.S.astype(np.float64), Vt


# ------------------------------------------------------------------------------------------
# Token routing.  [P1] "Delta-CoMe的应用场景" (multi-tenant serving: one dedicated model per
# customer on shared hardware); [P2] "Problem"/"Key results" (many deltas served on one GPU).
# Stable counting sort by tenant id, -1 (backbone only) first.  Parity: pinned against a stable
# library sort; bit-exact.
# ------------------------------------------------------------------------------------------
def route_tokens(tenant_ids, n_tenants: int):
    """Return (perm, inv_perm, segments).

    perm[j]     = original index of the token at sorted position j,
    inv_perm[i] = sorted position of original token i,
    segments    = [(tenant, start, length)] for every tenant >= 0 present, ascending tenant.
    """
    ids = [int(t) for t in tenant_ids]
    for t in ids:
        if t < -1 or t >= n_tenants:
            raise ValueError(f"tenant id {t} out of range")
    counts = [0] * (n_tenants + 1)
    for t in ids:
        counts[t + 1] += 1
    starts = [0] * (n_tenants + 1)
    acc = 0
    for b in range(n_tenants + 1):
        starts[b] = acc
        acc += counts[b]
    fill = list(starts)
    perm = [0] * len(ids)
    for i, t in enumerate(ids):
        perm[fill[t + 1]] = i
        fill[t + 1] += 1
    inv = [0] * len(ids)
    for j, i in enumerate(perm):
        inv[i] = j
    segs = [(b - 1, starts[b], counts[b]) for b in range(1, n_tenants + 1) if counts[b] > 0]
    return np.asarray(perm, dtype=np.int32), np.asarray(inv, dtype=np.int32), segs


# ------------------------------------------------------------------------------------------
# Evaluation.  y = W_base x + U_hat (S * (V_hat^T x)) per token with its own tenant (R5).
# [P2] "Problem" (serve many fine-tuned models cheaply from one backbone); the per-token form
# of the delta product follows from Delta_hat = U_hat diag(S) V_hat^T.  Parity: pinned against
# brute force with the explicit matrix, permutation invariance and special cases.
# ------------------------------------------------------------------------------------------
def delta_only(artefacts, x: np.ndarray, tenant_ids, rows=None) -> np.ndarray:
    """U_hat (S * (V_hat^T x_k)) for every token k (zero rows for tenant -1).

    ``artefacts`` maps tenant id -> Artefact (list or dict).  ``rows`` selects output rows.
    """
    x = np.asarray(x, dtype=np.float64)
    ids = np.asarray(tenant_ids)
    T = x.shape[0]
    if T == 0:
        return np.zeros((0, 0 if rows is None else len(rows)))
    first = artefacts[0] if isinstance(artefacts, (list, tuple)) else next(iter(artefacts.values()))
    n_rows = first.d_out if rows is None else len(rows)
    out = np.zeros((T, n_rows))
    for tau in sorted(set(int(t) for t in ids)):
        if tau < 0:
            continue
        a = artefacts[tau]
        ks = np.nonzero(ids == tau)[0]
        Uh, S, Vt = dequantized_factors(a, u_rows=rows)
        t = (Vt @ x[ks].T) * S[:, None]        # [r, n_tokens]
        out[ks] = (Uh @ t).T
    return out


def delta_linear(w_base: np.ndarray, artefacts, x: np.ndarray, tenant_ids, rows=None) -> np.ndarray:
    """y_k = W_base x_k + U_hat_tau (S_tau * (V_hat_tau^T x_k)), fp64 from exactly upcast inputs."""
    W = np.asarray(w_base, dtype=np.float64)
    if rows is not None:
        W = W[np.asarray(rows)] if W.shape[0] != len(rows) else W
    y = np.asarray(x, dtype=np.float64) @ W.T
    return y + delta_only(artefacts, x, tenant_ids, rows)


def brute_force_linear(w_base: np.ndarray, artefacts, x: np.ndarray, tenant_ids) -> np.ndarray:
    """Tiny inputs only: y_k = (W_base + U_hat diag(S) V_hat^T) x_k with the matrix formed."""
    W = np.asarray(w_base, dtype=np.float64)
    x = np.asarray(x, dtype=np.float64)
    y = np.zeros((x.shape[0], W.shape[0]))
    for k in range(x.shape[0]):
        tau = int(tenant_ids[k])
        M = W.copy()
        if tau >= 0:
            Uh, S, Vt = dequantized_factors(artefacts[tau])
            for i in range(S.shape[0]):
                M += S[i] * np.outer(Uh[:, i], Vt[i])
        for o in range(W.shape[0]):
            y[k, o] = float(np.dot(M[o], x[k]))
    return y


def activation_error(delta: np.ndarray, a: Artefact, x: np.ndarray) -> float:
    """||Delta X - Delta_hat X||_F / ||Delta X||_F over the tokens X (rows of x).

    [P2] "Experimental setup" names activation approximation error as a measured quantity.
    """
    D = np.asarray(delta, dtype=np.float64)
    X = np.asarray(x, dtype=np.float64)
    Uh, S, Vt = dequantized_factors(a)
    ref = X @ D.T
    approx = ((X @ Vt.T) * S[None, :]) @ Uh.T
    return float(np.linalg.norm(ref - approx) / np.linalg.norm(ref))
