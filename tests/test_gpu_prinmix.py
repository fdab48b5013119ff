"""Serving PrinMix-allocated deltas: widths chosen per rank by the 0/1 ILP over eq. 5 scores, U
refit by RTC, ranks regrouped into 8/3/2-bit bands ("Enhancing Delta Compression in LLMs via
SVD-based Quantization Error Minimization", sections 2.1-2.4).  The hot path is unchanged; the band
sizes become arbitrary (a band may be empty, the 3-bit band may be the largest), which exercises
the kernels' general band table.

The library's host routine (dc_prinmix_compress) produces the factors; the device serves them; the
fp64 oracle evaluates the same factors (and, independently, its own PrinMix compression of the
same SVD factors).
"""
import ctypes

import numpy as np
import pytest

import oracle
from oracle import prinmix as pm
import tenant_mixed_precision_b200 as dc
from tenant_mixed_precision_b200 import synth

from dc_testlib import assert_close

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu
if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("no CUDA device", allow_module_level=True)


@pytest.mark.parametrize("ratio,max_kinds", [(1 / 16, 3), (1 / 64, 2), (1 / 32, 1)])
def test_prinmix_tenants_served_against_oracle(ratio, max_kinds):
    rng = np.random.default_rng(int(1 / ratio) + max_kinds)
    d_out, d_in, n_ten, cand, n_cal = 512, 384, 3, 160, 256
    wb, wv = synth.bf16_round((0.02 * rng.standard_normal((d_out, d_in))).astype(np.float32))
    Xc = rng.standard_normal((n_cal, d_in)).astype(np.float32)  # calibration tokens
    handles, bufs, arts, arts_o = [], [], {}, {}
    for t in range(n_ten):
        U0, _ = np.linalg.qr(rng.standard_normal((d_out, cand)))
        V0, _ = np.linalg.qr(rng.standard_normal((d_in, cand)))
        S0 = (1.28 * np.arange(1, cand + 1) ** -0.8 * rng.uniform(0.5, 1.5, size=cand)).astype(np.float32)
        S0 = -np.sort(-S0)
        U0, Vt0 = U0.astype(np.float32), V0.T.astype(np.float32).copy()
        desc, perm, Uo, So, Vo, obj = dc.dc_prinmix_compress(U0, S0, Vt0, Xc, ratio, max_kinds)
        plan = [(desc.bits[i], desc.rank[i]) for i in range(desc.n_bands)]
        assert len(plan) <= max_kinds and sum(r for _, r in plan) > 0
        cu, cv, su, sv = dc.dc_quantize_rtn(desc, Uo, Vo)
        buf = torch.empty(dc.dc_packed_size(desc), dtype=torch.uint8, device="cuda")
        handles.append(dc.dc_pack_upload(desc, cu, cv, su, sv, So, buf))
        bufs.append(buf)
        arts[t] = oracle.compress_factors(Uo, So, Vo, plan)
        arts_o[t], _, _ = pm.compress_prinmix(U0, S0, Vt0, Xc, ratio, max_kinds)
    table = torch.empty(n_ten * ctypes.sizeof(dc.dc_delta_handle), dtype=torch.uint8, device="cuda")
    keep = dc.dc_tenant_table_upload(handles, table)
    max_rank = max(a.rank for a in arts.values())
    T = 12
    ids = np.array([t % n_ten for t in range(T)], dtype=np.int32)
    rng.shuffle(ids)
    xb, xv = synth.bf16_round(rng.standard_normal((T, d_in)).astype(np.float32))
    W = torch.from_numpy(wb.view(np.int16)).cuda().view(torch.bfloat16)
    x = torch.from_numpy(xb.view(np.int16)).cuda().view(torch.bfloat16)
    lin = dc.make_linear(W, d_out, d_in, n_ten, max_rank, table)
    ws = torch.zeros(dc.dc_workspace_size(T, max_rank, max(d_in, d_out), 1, n_ten), dtype=torch.uint8, device="cuda")
    xd = xv.astype(np.float64)
    for flags in (dc.DC_DELTA, dc.DC_BASE | dc.DC_DELTA):
        y = torch.full((T, d_out), float("nan"), dtype=torch.float32, device="cuda")
        dc.dc_delta_linear_segmented(lin, x, y, torch.from_numpy(ids).cuda(), T, flags, ws)
        torch.cuda.synchronize()
        assert dc.dc_read_device_status(ws) == 0
        got = y.cpu().numpy()
        want = oracle.delta_only(arts, xd, ids) + (xd @ wv.astype(np.float64).T if flags & dc.DC_BASE else 0)
        assert_close(got, want, f"PrinMix {ratio} K={max_kinds} flags={flags}")
        want_o = oracle.delta_only(arts_o, xd, ids) + (xd @ wv.astype(np.float64).T if flags & dc.DC_BASE else 0)
        assert_close(got, want_o, f"PrinMix vs the oracle's own compression {ratio} K={max_kinds} flags={flags}")
    del keep
