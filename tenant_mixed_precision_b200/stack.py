"""A multi-tenant linear stack on one GPU: the backbone's projections plus every tenant's packed
delta, served layer by layer through dc_layer_forward.

The stack owns (as torch tensors, i.e. caller-side device memory of the C library):
  * the bf16 backbone weights of every (layer, projection),
  * one arena holding every tenant's packed delta blob (256-byte aligned slices),
  * one device tenant table per (layer, projection),
  * the workspace, the per-layer inputs (x_h, x_o, x_f) and outputs.
forward() runs routing once and then the seven projections of every layer; it can be captured
in a CUDA graph.
"""
from __future__ import annotations

import ctypes as C

import torch

from . import (DC_BASE, DC_DELTA, DC_REUSE_ROUTING, dc_delta_handle, dc_layer_forward, dc_packed_size,
               dc_quantize_pack_device, dc_quantize_scratch_size, dc_tenant_table_upload, dc_workspace_size, make_desc,
               make_linear)
from .synth import PROJ_INPUT, llama_proj_shapes

HANDLE_BYTES = C.sizeof(dc_delta_handle)


def _align(x: int, a: int = 256) -> int:
    return (x + a - 1) // a * a


class DeltaStack:
    def __init__(self, hidden: int, ffn: int, layers: int, n_tenants: int, T_max: int, plan_fn,
                 out_dtype=torch.bfloat16, device: str = "cuda"):
        """plan_fn(layer, proj, d_out, d_in, tenant) -> [(bits, rank), ...] or None (no delta)."""
        self.hidden, self.ffn, self.layers, self.n_tenants, self.T_max = hidden, ffn, layers, n_tenants, T_max
        self.shapes = llama_proj_shapes(hidden, ffn)
        self.device = device
        self.descs = {}
        offsets = {}
        total = 0
        self.max_rank = [0] * 7
        for l in range(layers):
            for p, (d_out, d_in) in enumerate(self.shapes):
                for t in range(n_tenants):
                    plan = plan_fn(l, p, d_out, d_in, t)
                    if not plan:
                        continue
                    desc = make_desc(d_out, d_in, plan)
                    self.descs[(l, p, t)] = desc
                    offsets[(l, p, t)] = total
                    total += _align(dc_packed_size(desc))
                    self.max_rank[p] = max(self.max_rank[p], sum(r for b, r in plan if b))
        self.offsets = offsets
        self.arena = torch.empty(max(total, 256), dtype=torch.uint8, device=device)
        self.handles = {}
        self.W = [[torch.empty(s, dtype=torch.bfloat16, device=device) for s in self.shapes] for _ in range(layers)]
        self.tables = torch.zeros((layers, 7, max(1, n_tenants) * HANDLE_BYTES), dtype=torch.uint8, device=device)
        self.x = [[torch.zeros((T_max, d), dtype=torch.bfloat16, device=device) for d in (hidden, hidden, ffn)]
                  for _ in range(layers)]
        self.y = [[torch.zeros((T_max, s[0]), dtype=out_dtype, device=device) for s in self.shapes]
                  for _ in range(layers)]
        self.ws = torch.zeros(dc_workspace_size(T_max, max(self.max_rank), ffn, 7, n_tenants), dtype=torch.uint8,
                              device=device)
        self._lins = None
        self._keep = []
        self.fp8 = False

    def to_fp8_backbone(self, stream=None):
        """Replace every bf16 backbone weight by its E4M3 blob (codes, then fp32 row scales),
        quantised on the device, and rebuild the linear descriptors (DC_DTYPE_FP8)."""
        from . import dc_quantize_fp8_rows_device
        for l in range(self.layers):
            for p in range(7):
                self.W[l][p] = dc_quantize_fp8_rows_device(self.W[l][p], stream=stream)
        self.fp8 = True
        self.finalize()

    # -- loading -----------------------------------------------------------------------------
    def scratch_for(self, l: int, p: int, t: int) -> int:
        return dc_quantize_scratch_size(self.descs[(l, p, t)])

    def load_from_device_factors(self, l, p, t, U_dev, Vt_dev, S_dev, scratch, stream=None):
        """U_dev: float32 [r, d_out] (column i = u_i), Vt_dev: [r, d_in], S_dev: [r]; quantised and
        packed on the GPU into the tenant's arena slice."""
        desc = self.descs[(l, p, t)]
        off = self.offsets[(l, p, t)]
        h = dc_quantize_pack_device(desc, U_dev, Vt_dev, S_dev, self.arena, scratch, stream=stream, dst_offset=off,
                                    dst_bytes=dc_packed_size(desc))
        self.handles[(l, p, t)] = h
        return h

    def finalize(self):
        """Upload every (layer, projection) tenant table and build the linear descriptors."""
        torch.cuda.synchronize()
        self._lins = []
        for l in range(self.layers):
            lins = []
            for p, (d_out, d_in) in enumerate(self.shapes):
                hs = [self.handles.get((l, p, t), dc_delta_handle()) for t in range(self.n_tenants)]
                if self.n_tenants:
                    self._keep.append(dc_tenant_table_upload(hs, self.tables[l, p]))
                lins.append(make_linear(self.W[l][p], d_out, d_in, self.n_tenants, self.max_rank[p], self.tables[l, p]))
            self._lins.append(lins)
        torch.cuda.synchronize()
        self._keep = []

    # -- serving -----------------------------------------------------------------------------
    def forward(self, ids_dev, T: int, flags: int = DC_BASE | DC_DELTA, stream=None, reuse_routing=False):
        for l in range(self.layers):
            f = flags | (DC_REUSE_ROUTING if (l > 0 or reuse_routing) else 0)
            xh, xo, xf = self.x[l]
            dc_layer_forward(self._lins[l], xh, xo, xf, self.y[l], ids_dev, T, f, self.ws, stream=stream)

    # -- accounting ----------------------------------------------------------------------------
    def delta_bytes(self, l, p, t) -> dict:
        """Bytes of one tenant's blob split by the kernel that reads them."""
        from . import desc_rank  # local import keeps the module namespace small
        desc = self.descs[(l, p, t)]
        d_out, d_in = desc.d_out, desc.d_in
        r = desc_rank(desc)
        code_bits_v = sum(desc.bits[i] * desc.rank[i] for i in range(desc.n_bands)) * d_in
        code_bits_u = sum(desc.bits[i] * desc.rank[i] for i in range(desc.n_bands)) * d_out
        meta_v = r * (d_in // 128) * 4
        meta_u = r * (d_out // 128) * 4
        return {"v": code_bits_v // 8 + meta_v + 4 * r, "u": code_bits_u // 8 + meta_u}

    def algorithmic_bytes(self, tenant_ids) -> dict:
        """What one decode step must move: every backbone weight once, every distinct tenant's
        packed delta once per (layer, projection), activations and outputs once."""
        distinct = sorted(set(int(t) for t in tenant_ids if 0 <= int(t) < self.n_tenants))
        T = len(tenant_ids)
        out_es = self.y[0][0].element_size()
        v = u = w = act = 0
        for l in range(self.layers):
            for p, (d_out, d_in) in enumerate(self.shapes):
                w += (d_out * d_in + 4 * d_out) if self.fp8 else 2 * d_out * d_in
                act += T * (2 * d_in + out_es * d_out)
                for t in distinct:
                    if (l, p, t) in self.descs:
                        b = self.delta_bytes(l, p, t)
                        v += b["v"]
                        u += b["u"]
        return {"backbone": w, "delta_v": v, "delta_u": u, "activations": act, "total": w + v + u + act,
                "distinct_tenants": len(distinct)}


class PagedStack:
    """The tenants of a populated DeltaStack served from fewer device slots through the library's
    pager (dc_pager_*): frequently used tenants stay resident, long-tail ones are copied in from
    pinned host memory when a batch needs them.

    Each tenant's packed blobs for all (layer, projection) form one host image (256-byte aligned
    pieces); the stack owns the slot arena and its own device tenant tables, whose handles start
    with dev_base = 0 and are kept current by the pager.  Backbone weights, inputs, outputs and the
    workspace are those of `ref`.
    """

    def __init__(self, ref: DeltaStack, n_slots: int, keep_ref_arena: bool = True):
        from . import Pager, make_linear as _ml
        self.ref = ref
        self.n_slots = n_slots
        n_tab = ref.layers * 7
        self.images, self.blob_offsets = {}, {}
        sizes = []
        for t in range(ref.n_tenants):
            offs, size = [], 0
            for l in range(ref.layers):
                for p in range(7):
                    if (l, p, t) in ref.descs:
                        offs.append(size)
                        size += _align(dc_packed_size(ref.descs[(l, p, t)]))
                    else:
                        offs.append(-1)
            self.blob_offsets[t] = offs
            sizes.append(size)
        self.slot_bytes = _align(max(sizes + [256]))
        for t in range(ref.n_tenants):
            img = torch.empty(max(sizes[t], 256), dtype=torch.uint8, pin_memory=True)
            for l in range(ref.layers):
                for p in range(7):
                    o = self.blob_offsets[t][7 * l + p]
                    if o < 0:
                        continue
                    n = dc_packed_size(ref.descs[(l, p, t)])
                    src = ref.offsets[(l, p, t)]
                    img[o:o + n].copy_(ref.arena[src:src + n])
            self.images[t] = img
        torch.cuda.synchronize()
        self.arena = torch.empty(n_slots * self.slot_bytes, dtype=torch.uint8, device=ref.device)
        self.tables = torch.zeros_like(ref.tables)
        keep = []
        self.lins = []
        for l in range(ref.layers):
            lins = []
            for p, (d_out, d_in) in enumerate(ref.shapes):
                hs = []
                for t in range(ref.n_tenants):
                    h = ref.handles.get((l, p, t))
                    h2 = dc_delta_handle.from_buffer_copy(h) if h is not None else dc_delta_handle()
                    h2.dev_base = 0
                    hs.append(h2)
                if ref.n_tenants:
                    keep.append(dc_tenant_table_upload(hs, self.tables[l, p]))
                lins.append(_ml(ref.W[l][p], d_out, d_in, ref.n_tenants, ref.max_rank[p], self.tables[l, p]))
            self.lins.append(lins)
        torch.cuda.synchronize()
        del keep
        self.pager = Pager(ref.n_tenants, n_slots, self.slot_bytes, self.arena,
                           [self.tables[l, p] for l in range(ref.layers) for p in range(7)])
        for t in range(ref.n_tenants):
            self.pager.set_tenant(t, self.images[t], self.blob_offsets[t])
        if not keep_ref_arena:
            ref.arena = None

    def forward(self, ids_host, ids_dev, T: int, compute_stream, copy_stream, flags: int = DC_BASE | DC_DELTA):
        """Make the batch's tenants resident (copies on copy_stream), then run every layer on
        compute_stream, then mark the batch's slots as in use until those kernels finish."""
        self.pager.prepare(ids_host[:T], copy_stream, compute_stream)
        r = self.ref
        for l in range(r.layers):
            f = flags | (DC_REUSE_ROUTING if l > 0 else 0)
            xh, xo, xf = r.x[l]
            dc_layer_forward(self.lins[l], xh, xo, xf, r.y[l], ids_dev, T, f, r.ws, stream=compute_stream)
        self.pager.commit(compute_stream)

    def image_bytes(self, t: int) -> int:
        return self.images[t].numel()
