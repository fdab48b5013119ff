"""Fill a DeltaStack with the seeded synthetic workload (inputs only; no method arithmetic here).

Backbone weights ~ N(0, 0.02^2) bf16, tenant factors = Gaussian/sqrt(d) columns with the long-tail
spectrum s_i = s0 * i^-alpha, activations ~ N(0, 1) bf16, all drawn on the GPU from the same
counter-based stream that synth.py implements on the host, so the oracle can regenerate any
single matrix.  The factors are then quantised and packed by the library
(dc_quantize_pack_device).
"""
from __future__ import annotations

import math

import torch

from . import synth, synth_normal_device
from .stack import DeltaStack


def populate(stack: DeltaStack, seed: int, s0: float = 1.28, alpha: float = 0.8, T: int | None = None):
    T = stack.T_max if T is None else T
    dev = stack.device
    max_r = max(stack.max_rank) if stack.max_rank else 0
    max_d = max(stack.hidden, stack.ffn)
    u_buf = torch.empty(max(1, max_r * max_d), dtype=torch.float32, device=dev)
    v_buf = torch.empty(max(1, max_r * max_d), dtype=torch.float32, device=dev)
    scratch_bytes = max([stack.scratch_for(*k) for k in stack.descs] + [256])
    scratch = torch.zeros(scratch_bytes, dtype=torch.uint8, device=dev)
    spectra = {}
    for l in range(stack.layers):
        for p, (d_out, d_in) in enumerate(stack.shapes):
            synth_normal_device(stack.W[l][p], seed, synth.stream_id(0, l, p), 0, float(synth.ih4_scale(0.02)))
            for t in range(stack.n_tenants):
                if (l, p, t) not in stack.descs:
                    continue
                desc = stack.descs[(l, p, t)]
                r = sum(desc.rank[i] for i in range(desc.n_bands) if desc.bits[i])
                U = u_buf[: r * d_out]
                V = v_buf[: r * d_in]
                synth_normal_device(U, seed, synth.stream_id(1, l, p, t), 0,
                                    float(synth.ih4_scale(1.0 / math.sqrt(d_out))))
                synth_normal_device(V, seed, synth.stream_id(2, l, p, t), 0,
                                    float(synth.ih4_scale(1.0 / math.sqrt(d_in))))
                if r not in spectra:
                    spectra[r] = torch.from_numpy(synth.long_tail_spectrum(r, s0, alpha)).to(dev)
                stack.load_from_device_factors(l, p, t, U, V, spectra[r], scratch)
        for which, d in enumerate((stack.hidden, stack.hidden, stack.ffn)):
            synth_normal_device(stack.x[l][which][:T], seed, synth.stream_id(3, l, which), 0,
                                float(synth.ih4_scale(1.0)))
    torch.cuda.synchronize()
    status = int(scratch[:4].view(torch.int32).item())
    if status != 0:
        raise RuntimeError(f"device quantiser reported status {status}")
    stack.finalize()


def host_factors(seed: int, layer: int, proj: int, tenant: int, d_out: int, d_in: int, r: int,
                 s0: float = 1.28, alpha: float = 0.8):
    """The same factors populate() draws on the GPU, regenerated on the host (oracle input)."""
    return synth.stream_factors(seed, layer, proj, tenant, d_out, d_in, r, s0, alpha)


def host_activations(seed: int, layer: int, which: int, T: int, d: int):
    return synth.stream_activations(seed, layer, which, T, d)
