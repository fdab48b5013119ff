// Tenant paging over a device arena of fixed-size slots.
//
// "Delta-CoMe – 清华联合 OpenBMB 等高校开源的新型增量压缩算法", FAQ "多模型同机部署最该关注什么？":
// when many models share a machine, keep the frequently used ones resident and load the long-tail
// ones on demand.  Here every tenant's packed deltas (all of its linears) form one host image in
// pinned memory; the device holds at most n_slots of them.  Before a batch, dc_pager_prepare
// brings its missing tenants in (least recently used slots first, never a slot of the batch):
//   - on the copy stream: wait until the last batch that read the victim slot has finished, one
//     cudaMemcpyAsync of the whole image into the slot, then one small kernel that points the
//     tenant's handles in every tenant table at the slot (and the victim's at nothing);
//   - the compute stream waits for that copy stream work, so the batch's kernels see the tenants
//     in place, while copies for the next batch can overlap the current batch's kernels.
// dc_pager_commit, called after the batch's kernels are enqueued, records on the compute stream
// when the batch's slots are free again.  The library allocates no device memory: the arena, the
// tables and the patch scratch are the caller's.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstring>
#include <vector>

#include "dc.h"
#include "dc_internal.h"
#include "dc_lru.h"

namespace {

struct PatchRec {
  uint64_t addr;   // device address of a handle's dev_base
  uint64_t value;  // new dev_base (0: no delta)
};

__global__ void k_pager_patch(const PatchRec* __restrict__ recs, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) *reinterpret_cast<uint64_t*>(recs[i].addr) = recs[i].value;
}

struct TenantImage {
  const uint8_t* host = nullptr;
  uint64_t bytes = 0;
  std::vector<int64_t> offset;  // per table: blob offset inside the image, -1 = no blob
};

}  // namespace

struct dc_pager {
  dc_pager_desc d;
  uint8_t* arena = nullptr;
  std::vector<uint8_t*> tables;  // device tables [n_tenants] of dc_delta_handle
  PatchRec* scratch = nullptr;
  size_t scratch_recs = 0;
  std::vector<TenantImage> img;
  DcLru lru;
  std::vector<cudaEvent_t> slot_free;  // recorded on the compute stream after the last batch using the slot
  std::vector<char> slot_pending;      // slot_free has been recorded at least once
  cudaEvent_t ready = nullptr;
  std::vector<int32_t> batch_slots;    // slots of the batch being prepared (for commit)
  dc_pager_stats stats;
  dc_pager(const dc_pager_desc& dd) : d(dd), lru(dd.n_tenants, dd.n_slots) { std::memset(&stats, 0, sizeof(stats)); }
};

static size_t pager_scratch_recs(const dc_pager_desc* d) {
  // per batch: the loads (at most n_slots) each patch their tenant and their victim in every table
  return (size_t)2 * (size_t)d->n_slots * (size_t)d->n_tables;
}

extern "C" size_t dc_pager_scratch_size(const dc_pager_desc* d) {
  DC_NVTX("dc_pager_scratch_size");
  if (!d || d->n_slots <= 0 || d->n_tables <= 0) return 0;
  return pager_scratch_recs(d) * sizeof(PatchRec);
}

extern "C" dc_status dc_pager_create(const dc_pager_desc* d, void* arena_dev, size_t arena_bytes,
                                     void* const* tables_dev, void* scratch_dev, size_t scratch_bytes,
                                     dc_pager** out) {
  DC_NVTX("dc_pager_create");
  dc_clear_error();
  if (!d || !out || !arena_dev || !tables_dev || !scratch_dev) return dc_fail(DC_ERR_INVALID_ARG, "null argument");
  *out = nullptr;
  if (d->n_tenants <= 0 || d->n_slots <= 0 || d->n_tables <= 0 || d->slot_bytes == 0)
    return dc_fail(DC_ERR_INVALID_ARG, "pager: tenants, slots, tables and slot bytes must be positive");
  if (d->slot_bytes % 256) return dc_fail(DC_ERR_ALIGN, "pager: slot_bytes must be a multiple of 256");
  if (((uintptr_t)arena_dev & 255) != 0) return dc_fail(DC_ERR_ALIGN, "pager: arena must be 256-byte aligned");
  if (((uintptr_t)scratch_dev & 15) != 0) return dc_fail(DC_ERR_ALIGN, "pager: scratch must be 16-byte aligned");
  if (arena_bytes < (size_t)d->n_slots * d->slot_bytes)
    return dc_fail(DC_ERR_WORKSPACE, "pager: the arena holds %zu bytes, %d slots need %llu", arena_bytes,
                   d->n_slots, (unsigned long long)((uint64_t)d->n_slots * d->slot_bytes));
  if (scratch_bytes < dc_pager_scratch_size(d)) return dc_fail(DC_ERR_WORKSPACE, "pager: scratch too small");
  for (int i = 0; i < d->n_tables; ++i)
    if (!tables_dev[i] || ((uintptr_t)tables_dev[i] & 7) != 0)
      return dc_fail(DC_ERR_ALIGN, "pager: table %d is null or not 8-byte aligned", i);
  dc_pager* P = new dc_pager(*d);
  P->arena = (uint8_t*)arena_dev;
  P->tables.assign((uint8_t* const*)tables_dev, (uint8_t* const*)tables_dev + d->n_tables);
  P->scratch = (PatchRec*)scratch_dev;
  P->scratch_recs = pager_scratch_recs(d);
  P->img.resize(d->n_tenants);
  P->slot_free.assign(d->n_slots, nullptr);
  P->slot_pending.assign(d->n_slots, 0);
  cudaError_t e = cudaEventCreateWithFlags(&P->ready, cudaEventDisableTiming);
  for (int s = 0; s < d->n_slots && e == cudaSuccess; ++s)
    e = cudaEventCreateWithFlags(&P->slot_free[s], cudaEventDisableTiming);
  if (e != cudaSuccess) {
    dc_pager_destroy(P);
    return dc_cuda_check(e, "pager events");
  }
  *out = P;
  return DC_OK;
}

extern "C" dc_status dc_pager_set_tenant(dc_pager* P, int32_t tenant, const void* image_host, uint64_t image_bytes,
                                         const int64_t* blob_offsets) {
  DC_NVTX("dc_pager_set_tenant");
  dc_clear_error();
  if (!P || !image_host || !blob_offsets) return dc_fail(DC_ERR_INVALID_ARG, "null argument");
  if (tenant < 0 || tenant >= P->d.n_tenants) return dc_fail(DC_ERR_TENANT, "tenant %d out of range", tenant);
  if (image_bytes == 0 || image_bytes > P->d.slot_bytes)
    return dc_fail(DC_ERR_WORKSPACE, "pager: image of %llu bytes does not fit a slot of %llu",
                   (unsigned long long)image_bytes, (unsigned long long)P->d.slot_bytes);
  if (P->lru.slot_of(tenant) >= 0) return dc_fail(DC_ERR_INVALID_ARG, "pager: tenant %d is resident", tenant);
  for (int i = 0; i < P->d.n_tables; ++i) {
    const int64_t o = blob_offsets[i];
    if (o >= (int64_t)image_bytes || (o >= 0 && (o & 255)))
      return dc_fail(DC_ERR_INVALID_ARG, "pager: blob offset %lld outside the image or not 256-byte aligned",
                     (long long)o);
  }
  TenantImage& I = P->img[tenant];
  I.host = (const uint8_t*)image_host;
  I.bytes = image_bytes;
  I.offset.assign(blob_offsets, blob_offsets + P->d.n_tables);
  return DC_OK;
}

extern "C" dc_status dc_pager_prepare(dc_pager* P, const int32_t* tenant_ids_host, int32_t T, void* copy_stream,
                                      void* compute_stream) {
  DC_NVTX("dc_pager_prepare");
  dc_clear_error();
  if (!P || (T > 0 && !tenant_ids_host)) return dc_fail(DC_ERR_INVALID_ARG, "null argument");
  if (T < 0) return dc_fail(DC_ERR_INVALID_ARG, "negative T");
  cudaStream_t cs = (cudaStream_t)copy_stream, ks = (cudaStream_t)compute_stream;
  std::vector<char> seen(P->d.n_tenants, 0);
  std::vector<int32_t> distinct;
  for (int i = 0; i < T; ++i) {
    const int32_t t = tenant_ids_host[i];
    if (t < 0) continue;  // backbone only
    if (t >= P->d.n_tenants) return dc_fail(DC_ERR_TENANT, "tenant id %d out of range", t);
    if (!seen[t]) {
      seen[t] = 1;
      distinct.push_back(t);
    }
  }
  for (int32_t t : distinct)
    if (!P->img[t].host) return dc_fail(DC_ERR_INVALID_ARG, "pager: tenant %d has no image", t);
  std::vector<DcLru::Load> loads;
  if (!P->lru.plan(distinct, loads, P->stats.hits, P->stats.misses))
    return dc_fail(DC_ERR_UNSUPPORTED, "pager: the batch holds %zu tenants, more than the %d slots",
                   distinct.size(), P->d.n_slots);
  P->batch_slots.clear();
  for (int32_t t : distinct) P->batch_slots.push_back(P->lru.slot_of(t));
  P->stats.batches += 1;
  if (loads.empty()) return DC_OK;  // everything resident: nothing for the compute stream to wait on
  std::vector<PatchRec> recs;
  dc_status st = DC_OK;
  for (const DcLru::Load& L : loads) {
    uint8_t* dst = P->arena + (size_t)L.slot * P->d.slot_bytes;
    if (P->slot_pending[L.slot])  // the last batch that read this slot must have finished
      st = dc_cuda_check(cudaStreamWaitEvent(cs, P->slot_free[L.slot], 0), "pager wait");
    if (st) return st;
    const TenantImage& I = P->img[L.tenant];
    st = dc_cuda_check(cudaMemcpyAsync(dst, I.host, I.bytes, cudaMemcpyHostToDevice, cs), "pager image copy");
    if (st) return st;
    P->stats.bytes_loaded += (int64_t)I.bytes;
    for (int i = 0; i < P->d.n_tables; ++i) {
      const uint64_t hoff = (uint64_t)L.tenant * sizeof(dc_delta_handle) + offsetof(dc_delta_handle, dev_base);
      if (L.evicted >= 0) {
        const uint64_t voff = (uint64_t)L.evicted * sizeof(dc_delta_handle) + offsetof(dc_delta_handle, dev_base);
        recs.push_back(PatchRec{(uint64_t)(uintptr_t)(P->tables[i] + voff), 0});
      }
      const int64_t o = I.offset[i];
      recs.push_back(PatchRec{(uint64_t)(uintptr_t)(P->tables[i] + hoff), o >= 0 ? (uint64_t)(uintptr_t)(dst + o) : 0});
    }
    if (L.evicted >= 0) P->stats.evictions += 1;
  }
  if (recs.size() > P->scratch_recs) return dc_fail(DC_ERR_WORKSPACE, "pager: patch scratch too small");
  // pageable source: the call returns once the records are staged, so `recs` may go out of scope
  st = dc_cuda_check(cudaMemcpyAsync(P->scratch, recs.data(), recs.size() * sizeof(PatchRec), cudaMemcpyHostToDevice, cs),
                     "pager patch upload");
  if (st) return st;
  const int n = (int)recs.size();
  k_pager_patch<<<(n + 255) / 256, 256, 0, cs>>>(P->scratch, n);
  st = dc_cuda_check(cudaGetLastError(), "pager patch kernel");
  if (st) return st;
  st = dc_cuda_check(cudaEventRecord(P->ready, cs), "pager ready event");
  if (st) return st;
  return dc_cuda_check(cudaStreamWaitEvent(ks, P->ready, 0), "pager compute wait");
}

extern "C" dc_status dc_pager_commit(dc_pager* P, void* compute_stream) {
  DC_NVTX("dc_pager_commit");
  dc_clear_error();
  if (!P) return dc_fail(DC_ERR_INVALID_ARG, "null pager");
  for (int32_t s : P->batch_slots) {
    dc_status st = dc_cuda_check(cudaEventRecord(P->slot_free[s], (cudaStream_t)compute_stream), "pager slot event");
    if (st) return st;
    P->slot_pending[s] = 1;
  }
  P->batch_slots.clear();
  return DC_OK;
}

extern "C" dc_status dc_pager_get_stats(const dc_pager* P, dc_pager_stats* out) {
  DC_NVTX("dc_pager_get_stats");
  dc_clear_error();
  if (!P || !out) return dc_fail(DC_ERR_INVALID_ARG, "null argument");
  *out = P->stats;
  return DC_OK;
}

extern "C" int32_t dc_pager_slot_of(const dc_pager* P, int32_t tenant) {
  DC_NVTX("dc_pager_slot_of"); return P ? P->lru.slot_of(tenant) : -1; }

extern "C" dc_status dc_pager_destroy(dc_pager* P) {
  DC_NVTX("dc_pager_destroy");
  dc_clear_error();
  if (!P) return DC_OK;
  if (P->ready) cudaEventDestroy(P->ready);
  for (cudaEvent_t e : P->slot_free)
    if (e) cudaEventDestroy(e);
  delete P;
  return DC_OK;
}
