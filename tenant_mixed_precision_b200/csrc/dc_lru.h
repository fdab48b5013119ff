// Residency policy of the tenant pager: which tenants occupy the device slots, and which slot a
// missing tenant takes.
//
// Frequently used tenants stay resident and long-tail tenants are loaded on demand ("Delta-CoMe –
// 清华联合 OpenBMB 等高校开源的新型增量压缩算法", FAQ "多模型同机部署最该关注什么？": keep the common
// models resident, load the long-tail ones when asked for).  The policy is least-recently-used over
// batches: every tenant of a batch is stamped with the batch's number; a missing tenant takes a free
// slot, else the slot whose tenant has the oldest stamp, never one stamped by the current batch.
// Plain C++ with no CUDA types, so that it can be checked on a machine without a GPU.
#pragma once
#include <stdint.h>

#include <vector>

class DcLru {
 public:
  struct Load {
    int32_t tenant;   // tenant to bring in
    int32_t slot;     // slot it takes
    int32_t evicted;  // tenant that held the slot (-1 if the slot was free)
  };

  DcLru(int32_t n_tenants, int32_t n_slots)
      : slot_of_(n_tenants, -1), stamp_(n_tenants, 0), tenant_in_(n_slots, -1) {}

  int32_t n_tenants() const { return (int32_t)slot_of_.size(); }
  int32_t n_slots() const { return (int32_t)tenant_in_.size(); }
  int32_t slot_of(int32_t t) const { return t >= 0 && t < n_tenants() ? slot_of_[t] : -1; }
  int32_t tenant_in(int32_t s) const { return s >= 0 && s < n_slots() ? tenant_in_[s] : -1; }

  // Plan one batch over its distinct tenants (each in range, no repeats).  Stamps every tenant of
  // the batch, returns the loads for the missing ones in `loads` and counts hits and misses.
  // Returns false (and changes nothing) if the batch holds more tenants than there are slots.
  bool plan(const std::vector<int32_t>& distinct, std::vector<Load>& loads, int64_t& hits, int64_t& misses) {
    loads.clear();
    if ((int64_t)distinct.size() > (int64_t)n_slots()) return false;
    const uint64_t now = ++clock_;
    for (int32_t t : distinct) stamp_[t] = now;
    for (int32_t t : distinct) {
      if (slot_of_[t] >= 0) {
        ++hits;
        continue;
      }
      ++misses;
      int32_t best = -1;
      uint64_t best_stamp = 0;
      for (int32_t s = 0; s < n_slots(); ++s) {
        const int32_t v = tenant_in_[s];
        if (v < 0) {  // a free slot wins at once
          best = s;
          break;
        }
        if (stamp_[v] == now) continue;  // in this batch
        if (best < 0 || stamp_[v] < best_stamp) {
          best = s;
          best_stamp = stamp_[v];
        }
      }
      // best >= 0: the batch has no more tenants than slots, and each of its resident tenants
      // holds one slot, so a slot outside the batch exists
      const int32_t v = tenant_in_[best];
      if (v >= 0) slot_of_[v] = -1;
      tenant_in_[best] = t;
      slot_of_[t] = best;
      loads.push_back(Load{t, best, v});
    }
    return true;
  }

 private:
  std::vector<int32_t> slot_of_;
  std::vector<uint64_t> stamp_;
  std::vector<int32_t> tenant_in_;
  uint64_t clock_ = 0;
};
