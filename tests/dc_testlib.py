"""Helpers shared by the GPU tests: upload tenants through the C ABI, compare with the oracle."""
from __future__ import annotations

import math

import numpy as np

import oracle
import tenant_mixed_precision_b200 as dc
from tenant_mixed_precision_b200 import synth

# Tolerances stated for the serving path: relative L2 error <= 1e-3 and max abs error <= 1e-2 * max|y|.
REL_L2 = 1e-3
MAX_ABS_FRAC = 1e-2


def rel_l2(a, b) -> float:
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    den = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / den) if den > 0 else float(np.linalg.norm(a - b))


def assert_close(got, ref, what=""):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    e = rel_l2(got, ref)
    m = float(np.max(np.abs(got - ref))) if got.size else 0.0
    lim = MAX_ABS_FRAC * float(np.max(np.abs(ref))) if ref.size else 0.0
    assert e <= REL_L2, f"{what}: relative L2 error {e:.3e} > {REL_L2}"
    assert m <= lim + 1e-30, f"{what}: max abs error {m:.3e} > {lim:.3e}"


class Guarded:
    """A device buffer with guard bytes on both sides -- the stand-in for a memory sanitizer, which
    is not available on the GPU pool.  The library gets the interior (4096 bytes in, so every
    alignment rule holds); check() asserts that no byte of either guard changed, i.e. that the
    kernels wrote nothing outside the buffer they were given."""

    GUARD = 4096
    PATTERN = 0xA5

    def __init__(self, torch, shape, dtype, fill=None):
        self.torch = torch
        n = 1
        for d in shape:
            n *= int(d)
        esz = torch.empty(0, dtype=dtype).element_size()
        self.nbytes = n * esz
        self.raw = torch.full((self.nbytes + 2 * self.GUARD,), self.PATTERN, dtype=torch.uint8, device="cuda")
        self.t = self.raw[self.GUARD:self.GUARD + self.nbytes].view(dtype).view(*shape)
        if fill is not None:
            self.t.fill_(fill)

    def check(self, what=""):
        self.torch.cuda.synchronize()
        head = self.raw[:self.GUARD]
        tail = self.raw[self.GUARD + self.nbytes:]
        bad = int((head != self.PATTERN).sum().item()) + int((tail != self.PATTERN).sum().item())
        assert bad == 0, f"{what}: {bad} guard bytes around the buffer were overwritten"


def gaussian_factors(rng, d_out, d_in, r, s0=1.28, alpha=0.8):
    U = (rng.standard_normal((d_out, r)) / math.sqrt(d_out)).astype(np.float32)
    Vt = (rng.standard_normal((r, d_in)) / math.sqrt(d_in)).astype(np.float32)
    S = synth.long_tail_spectrum(r, s0, alpha)
    return synth.Factors(np.asfortranarray(U), S, Vt)


class TenantDeltas:
    """Deltas of several tenants for one linear, quantised and packed through the C ABI.

    ``factors[t]`` is a synth.Factors or None (tenant without a delta).  The oracle artefacts of
    the same factors are kept in ``artefacts`` (None for tenants without a delta).
    """

    def __init__(self, torch, d_out, d_in, factors, plans, device_quantizer=False):
        self.d_out, self.d_in = d_out, d_in
        self.handles, self.buffers, self.artefacts, self.codes = [], [], [], []
        self.max_rank = 0
        for f, plan in zip(factors, plans):
            if f is None:
                self.handles.append(dc.empty_handle())
                self.artefacts.append(None)
                self.codes.append(None)
                continue
            desc = dc.make_desc(d_out, d_in, plan)
            r = dc.desc_rank(desc)
            U, S, Vt = f.U[:, :r], f.S[:r], f.Vt[:r]
            buf = torch.empty(dc.dc_packed_size(desc), dtype=torch.uint8, device="cuda")
            if device_quantizer:
                Ud = torch.from_numpy(np.ascontiguousarray(np.asarray(U, np.float32).T)).cuda()
                Vd = torch.from_numpy(np.ascontiguousarray(Vt, np.float32)).cuda()
                Sd = torch.from_numpy(np.ascontiguousarray(S, np.float32)).cuda()
                scratch = torch.zeros(dc.dc_quantize_scratch_size(desc), dtype=torch.uint8, device="cuda")
                h = dc.dc_quantize_pack_device(desc, Ud, Vd, Sd, buf, scratch)
                torch.cuda.synchronize()
                assert dc.dc_read_device_status(scratch) == 0
                self.codes.append(None)
            else:
                cu, cv, su, sv = dc.dc_quantize_rtn(desc, U, Vt)
                h = dc.dc_pack_upload(desc, cu, cv, su, sv, S, buf)
                self.codes.append((cu, cv, su, sv))
            self.handles.append(h)
            self.buffers.append(buf)
            self.artefacts.append(oracle.compress_factors(U, S, Vt, plan))
            self.max_rank = max(self.max_rank, r)
        import ctypes
        self.table = torch.empty(max(1, len(self.handles)) * ctypes.sizeof(dc.dc_delta_handle), dtype=torch.uint8,
                                 device="cuda")
        self._keep = dc.dc_tenant_table_upload(self.handles, self.table)
        torch.cuda.synchronize()

    def linear(self, W_base):
        return dc.make_linear(W_base, self.d_out, self.d_in, len(self.handles), self.max_rank, self.table)

    def oracle_artefacts(self):
        return {t: a for t, a in enumerate(self.artefacts) if a is not None}


def oracle_y(w_base_f64, td: TenantDeltas, x_f64, ids, flags):
    arts = td.oracle_artefacts()
    ids_eff = np.array([t if (t >= 0 and td.artefacts[t] is not None) else -1 for t in ids], dtype=np.int32)
    y = np.zeros((x_f64.shape[0], td.d_out))
    if flags & dc.DC_BASE:
        y += x_f64 @ w_base_f64.T
    if flags & dc.DC_DELTA and arts:
        y += oracle.delta_only(arts, x_f64, ids_eff)
    return y
