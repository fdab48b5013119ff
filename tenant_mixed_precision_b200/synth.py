"""Seeded synthetic inputs shared by the oracle tests, the GPU tests and the benchmark.

This module only draws numbers.  It holds none of the method's arithmetic: no SVD, no bit
allocation, no quantisation, no evaluation.  Everything it returns is an *input* (backbone
weights, fine-tuned deltas given as factors or as full matrices, activations, tenant ids) and
both sides of every parity check receive the same arrays.

Two kinds of generator live here:

* ``numpy.random.default_rng(seed)`` for the small workloads whose recipe fixes it (the single
  512x512 linear, the one-layer 7B batch, the tiny brute-force cases);
* a counter-based stream for the full-size workloads, so that a GPU kernel can produce the
  same numbers on the device (its CUDA twin is ``csrc/synth/synth_gen.cu``) and the oracle can
  regenerate any single matrix on the host.  The stream is SplitMix64 (Steele, Lea and Flood,
  "Fast splittable pseudorandom number generators", OOPSLA 2014): state_i = key + (i+1)*GAMMA,
  output = mix64(state_i).  A normal-like value takes the four 16-bit fields h0..h3 of one
  output and forms the centred Irwin-Hall(4) sum (h0+h1+h2+h3+2-2**17)/2**16, which has mean 0
  and variance 1/3; it is scaled by an fp32 constant c = fp32(sqrt(3)*sigma) with one fp32
  multiply (round to nearest even), so every value is reproducible bit for bit on any IEEE
  machine.

The spectra of the synthetic deltas follow the long-tail shape that the Delta-CoMe pages
describe (a few large singular values, many small ones): s_i = s0 * i**(-alpha).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

# ----------------------------------------------------------------------------------------
# bf16 helpers (numpy has no bf16 dtype; bf16 values are carried as their uint16 bit patterns
# plus the exactly equal float32 values)
# ----------------------------------------------------------------------------------------

def bf16_round(x) -> tuple[np.ndarray, np.ndarray]:
    """Round float32 values to bf16 (round to nearest, ties to even).

    Returns (bits uint16, values float32) where ``values`` are exactly the bf16 numbers.
    NaN is not expected in synthetic inputs and is not treated specially.
    """
    f = np.ascontiguousarray(x, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    r = (u + np.uint64(0x7FFF) + lsb) >> np.uint64(16)
    bits = r.astype(np.uint16)
    vals = (bits.astype(np.uint32) << np.uint32(16)).view(np.float32)
    return bits, vals


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


# ----------------------------------------------------------------------------------------
# SplitMix64 counter-based stream
# ----------------------------------------------------------------------------------------
GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)


def mix64(z: np.ndarray) -> np.ndarray:
    """SplitMix64 output function (variant 13 of Stafford's mixers, as published)."""
    z = np.asarray(z, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def stream_key(seed: int, stream: int) -> np.uint64:
    """Initial SplitMix64 state of stream ``stream`` under ``seed``."""
    with np.errstate(over="ignore"):
        a = mix64(np.uint64(seed & 0xFFFFFFFFFFFFFFFF) + GAMMA)
        b = mix64(a ^ (np.uint64(stream & 0xFFFFFFFFFFFFFFFF) + GAMMA + GAMMA))
    return np.uint64(b)


def stream_words(seed: int, stream: int, start: int, count: int) -> np.ndarray:
    key = stream_key(seed, stream)
    idx = np.arange(start + 1, start + count + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        return mix64(key + idx * GAMMA)


def ih4_scale(sigma: float) -> np.float32:
    """fp32 multiplier turning the Irwin-Hall(4) sum into a value of standard deviation sigma."""
    return np.float32(math.sqrt(3.0) * sigma)


def stream_normal(seed: int, stream: int, start: int, count: int, sigma: float) -> np.ndarray:
    """``count`` normal-like float32 values (elements start..start+count-1 of the stream)."""
    w = stream_words(seed, stream, start, count)
    m = np.uint64(0xFFFF)
    s = ((w & m) + ((w >> np.uint64(16)) & m) + ((w >> np.uint64(32)) & m) + (w >> np.uint64(48))).astype(np.int64)
    base = ((s + 2 - (1 << 17)).astype(np.float32)) * np.float32(1.0 / 65536.0)  # exact
    return (base * ih4_scale(sigma)).astype(np.float32)


# Stream identifiers for the full-size linear stacks.  kind: 0 = backbone weight, 1 = U
# factor, 2 = V factor (stored as V^T rows), 3 = activations.
def stream_id(kind: int, layer: int = 0, proj: int = 0, tenant: int = 0) -> int:
    return (((kind * 1024 + layer) * 16 + proj) * 4096) + tenant


# ----------------------------------------------------------------------------------------
# Shapes of the workloads
# ----------------------------------------------------------------------------------------
PROJ_NAMES = ("q", "k", "v", "o", "gate", "up", "down")


def llama_proj_shapes(hidden: int, ffn: int) -> list[tuple[int, int]]:
    """(d_out, d_in) of the seven projections of one Llama-style decoder layer."""
    return [(hidden, hidden)] * 4 + [(ffn, hidden)] * 2 + [(hidden, ffn)]


LLAMA7B = dict(hidden=4096, ffn=11008, layers=32)
LLAMA13B = dict(hidden=5120, ffn=13824, layers=40)

# Projection p reads input 0 (x_h), 1 (x_o) or 2 (x_f).
PROJ_INPUT = (0, 0, 0, 1, 0, 0, 2)


def long_tail_spectrum(r: int, s0: float, alpha: float) -> np.ndarray:
    """s_i = s0 * i**(-alpha), i = 1..r, rounded once to float32."""
    i = np.arange(1, r + 1, dtype=np.float64)
    return (s0 * i ** (-alpha)).astype(np.float32)


# ----------------------------------------------------------------------------------------
# The single 512x512 fp32 linear with two tenants
# ----------------------------------------------------------------------------------------
@dataclass
class SingleLinearCase:
    w_base: np.ndarray            # float32 [d_out, d_in]
    w_ft: list                    # float32 [d_out, d_in] per tenant (fine-tuned weights)
    x: np.ndarray                 # float32 [T, d_in]
    tenant_ids: np.ndarray        # int32 [T]
    plan: list = field(default_factory=list)   # [(bits, rank), ...] in singular-value order


def random_orthonormal(rng: np.random.Generator, n: int, k: int) -> np.ndarray:
    """n x k matrix with orthonormal columns: Q of the QR factorisation of a Gaussian matrix."""
    q, r = np.linalg.qr(rng.standard_normal((n, k)))
    return q * np.sign(np.diag(r))[None, :]


def single_linear_case(seed: int = 0, d: int = 512, n_tenants: int = 2, tokens_per_tenant: int = 2,
                       plan=((8, 2), (3, 8), (2, 32))) -> SingleLinearCase:
    rng = np.random.default_rng(seed)
    w_base = (0.02 * rng.standard_normal((d, d))).astype(np.float32)
    s = 0.05 / np.arange(1, d + 1, dtype=np.float64)
    w_ft = []
    for _ in range(n_tenants):
        q1 = random_orthonormal(rng, d, d)
        q2 = random_orthonormal(rng, d, d)
        delta = (q1 * s[None, :]) @ q2.T + 1e-4 * rng.standard_normal((d, d))
        w_ft.append((w_base.astype(np.float64) + delta).astype(np.float32))
    T = n_tenants * tokens_per_tenant
    x = rng.standard_normal((T, d)).astype(np.float32)
    tenant_ids = rng.permutation(np.repeat(np.arange(n_tenants, dtype=np.int32), tokens_per_tenant))
    return SingleLinearCase(w_base, w_ft, x, tenant_ids.astype(np.int32), [tuple(p) for p in plan])


# ----------------------------------------------------------------------------------------
# Factor-form deltas (closed-form SVD: Q1 diag(s) Q2^T with orthonormal Q's)
# ----------------------------------------------------------------------------------------
@dataclass
class Factors:
    U: np.ndarray    # float32 [d_out, r]  (column i = u_i)
    S: np.ndarray    # float32 [r]
    Vt: np.ndarray   # float32 [r, d_in]   (row i = v_i^T)


def qr_factors(rng: np.random.Generator, d_out: int, d_in: int, r: int, s0: float, alpha: float) -> Factors:
    q1 = random_orthonormal(rng, d_out, r)
    q2 = random_orthonormal(rng, d_in, r)
    return Factors(np.asfortranarray(q1.astype(np.float32)), long_tail_spectrum(r, s0, alpha),
                   np.ascontiguousarray(q2.T.astype(np.float32)))


def stream_factors(seed: int, layer: int, proj: int, tenant: int, d_out: int, d_in: int, r: int,
                   s0: float, alpha: float) -> Factors:
    """Gaussian/sqrt(d) columns from the counter-based stream (the full-size recipe)."""
    u = stream_normal(seed, stream_id(1, layer, proj, tenant), 0, d_out * r, 1.0 / math.sqrt(d_out))
    v = stream_normal(seed, stream_id(2, layer, proj, tenant), 0, r * d_in, 1.0 / math.sqrt(d_in))
    return Factors(np.asfortranarray(u.reshape(r, d_out).T), long_tail_spectrum(r, s0, alpha),
                   v.reshape(r, d_in))


def stream_base_weight(seed: int, layer: int, proj: int, d_out: int, d_in: int, rows=None):
    """bf16 backbone weight N(0, 0.02^2) from the counter-based stream; optionally a row subset."""
    sid = stream_id(0, layer, proj)
    if rows is None:
        vals = stream_normal(seed, sid, 0, d_out * d_in, 0.02).reshape(d_out, d_in)
    else:
        vals = np.stack([stream_normal(seed, sid, int(o) * d_in, d_in, 0.02) for o in rows])
    return bf16_round(vals)


def stream_activations(seed: int, layer: int, which: int, T: int, d: int):
    """bf16 activations N(0, 1) [T, d] from the counter-based stream."""
    vals = stream_normal(seed, stream_id(3, layer, which), 0, T * d, 1.0).reshape(T, d)
    return bf16_round(vals)


# ----------------------------------------------------------------------------------------
# Token -> tenant draws
# ----------------------------------------------------------------------------------------

def uniform_tenants(rng: np.random.Generator, T: int, n_tenants: int) -> np.ndarray:
    return rng.integers(0, n_tenants, size=T).astype(np.int32)


def zipf_tenants(rng: np.random.Generator, T: int, n_tenants: int, a: float = 1.1) -> np.ndarray:
    """Truncated Zipf popularity: P(tenant k-1) proportional to k**(-a), k = 1..n_tenants."""
    p = np.arange(1, n_tenants + 1, dtype=np.float64) ** (-a)
    p /= p.sum()
    return rng.choice(n_tenants, size=T, p=p).astype(np.int32)


def prefill_segments(rng: np.random.Generator, T: int, n_tenants: int, lo: int = 32, hi: int = 256) -> np.ndarray:
    """Tenant id per token for a prefill batch made of runs of lengths U{lo..hi}.

    Runs are drawn until T tokens are covered; the last run is cut to reach exactly T.
    Repeated tenants are allowed (the segment builder merges them).
    """
    ids = []
    while len(ids) < T:
        n = int(rng.integers(lo, hi + 1))
        t = int(rng.integers(0, n_tenants))
        ids.extend([t] * n)
    return np.asarray(ids[:T], dtype=np.int32)
