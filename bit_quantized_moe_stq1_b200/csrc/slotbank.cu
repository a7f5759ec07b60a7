// Expert slot bank (host side): routed experts live outside HBM and a fixed number of HBM
// slots hold the ones in use ("Hy4-preview-FlashMoE-STQ1_0", running with a slot bank:
// the routed tensors are read into the bank on demand, a miss reads its expert in, N slots
// hold N experts of a layer, and at least top-k slots are needed).  The pages do not state
// a replacement rule; this bank evicts the least recently used slot among those the
// current call does not need, ties to the lowest slot index.  A call then runs the MoE
// kernels with E = the slot count and every routed id replaced by its slot.

#include <cuda_runtime.h>

#include <cstdint>
#include <new>
#include <vector>

#include "common.cuh"

struct stq_slot_bank {
  int32_t n_experts = 0, n_slots = 0;
  int64_t clock = 0;                 // calls mapped so far
  std::vector<int32_t> slot_expert;  // [n_slots]: resident expert, -1 = empty
  std::vector<int64_t> slot_used;    // [n_slots]: clock of the last call that used the slot
  std::vector<int32_t> expert_slot;  // [n_experts]: slot holding the expert, -1 = not resident
};

extern "C" stq_slot_bank* stq_slot_bank_create(int32_t n_experts, int32_t n_slots) {
  if (n_experts <= 0 || n_slots <= 0 || n_slots > n_experts) return nullptr;
  stq_slot_bank* b = new (std::nothrow) stq_slot_bank();
  if (b == nullptr) return nullptr;
  b->n_experts = n_experts;
  b->n_slots = n_slots;
  b->slot_expert.assign(size_t(n_slots), -1);
  b->slot_used.assign(size_t(n_slots), -1);
  b->expert_slot.assign(size_t(n_experts), -1);
  return b;
}

extern "C" void stq_slot_bank_destroy(stq_slot_bank* b) { delete b; }

extern "C" stq_status stq_slot_bank_map(stq_slot_bank* b, const int32_t* ids, int64_t n, int32_t* slot_ids,
                                        int32_t* load_expert, int32_t* load_slot, int32_t* n_loads) {
  STQ_HOST_CHECK(b != nullptr && n >= 0 && n_loads != nullptr, STQ_ERR_INVALID_ARG);
  STQ_HOST_CHECK(n == 0 || (ids != nullptr && slot_ids != nullptr && load_expert != nullptr && load_slot != nullptr),
                 STQ_ERR_INVALID_ARG);
  // validate and collect the distinct experts in first-use order before touching the bank
  std::vector<char> seen(size_t(b->n_experts), 0);
  std::vector<int32_t> distinct;
  for (int64_t i = 0; i < n; ++i) {
    const int32_t e = ids[i];
    STQ_HOST_CHECK(e >= 0 && e < b->n_experts, STQ_ERR_INVALID_ARG);
    if (!seen[size_t(e)]) {
      seen[size_t(e)] = 1;
      distinct.push_back(e);
    }
  }
  STQ_HOST_CHECK(int64_t(distinct.size()) <= int64_t(b->n_slots), STQ_ERR_INVALID_ARG);
  const int64_t now = b->clock++;
  // hits first: mark their slots as used by this call, so no miss can evict them
  for (int32_t e : distinct) {
    const int32_t s = b->expert_slot[size_t(e)];
    if (s >= 0) b->slot_used[size_t(s)] = now;
  }
  int32_t loads = 0;
  for (int32_t e : distinct) {
    if (b->expert_slot[size_t(e)] >= 0) continue;
    // least recently used slot not used by this call (empty slots have clock -1)
    int32_t victim = -1;
    for (int32_t s = 0; s < b->n_slots; ++s) {
      if (b->slot_used[size_t(s)] == now) continue;
      if (victim < 0 || b->slot_used[size_t(s)] < b->slot_used[size_t(victim)]) victim = s;
    }
    // distinct <= n_slots guarantees a victim
    const int32_t old = b->slot_expert[size_t(victim)];
    if (old >= 0) b->expert_slot[size_t(old)] = -1;
    b->slot_expert[size_t(victim)] = e;
    b->expert_slot[size_t(e)] = victim;
    b->slot_used[size_t(victim)] = now;
    load_expert[loads] = e;
    load_slot[loads] = victim;
    ++loads;
  }
  for (int64_t i = 0; i < n; ++i) slot_ids[i] = b->expert_slot[size_t(ids[i])];
  *n_loads = loads;
  return STQ_OK;
}

extern "C" stq_status stq_slot_bank_resident(const stq_slot_bank* b, int32_t* slot_expert) {
  STQ_HOST_CHECK(b != nullptr && slot_expert != nullptr, STQ_ERR_INVALID_ARG);
  for (int32_t s = 0; s < b->n_slots; ++s) slot_expert[s] = b->slot_expert[size_t(s)];
  return STQ_OK;
}

extern "C" stq_status stq_slot_bank_copy(const stq_slot_bank* b, const int32_t* load_expert, const int32_t* load_slot,
                                         int32_t n_loads, int32_t n_mats, const void* const* src, void* const* dst,
                                         const size_t* mat_bytes, stq_stream_t stream) {
  STQ_HOST_CHECK(b != nullptr && n_loads >= 0 && n_mats >= 0, STQ_ERR_INVALID_ARG);
  if (n_loads == 0 || n_mats == 0) return STQ_OK;
  STQ_HOST_CHECK(load_expert != nullptr && load_slot != nullptr && src != nullptr && dst != nullptr &&
                     mat_bytes != nullptr,
                 STQ_ERR_INVALID_ARG);
  for (int32_t m = 0; m < n_mats; ++m) STQ_HOST_CHECK(src[m] != nullptr && dst[m] != nullptr, STQ_ERR_INVALID_ARG);
  // the arrays hold the bank's n_experts (source) and n_slots (destination) matrices: an
  // index outside them is refused before any copy is enqueued
  for (int32_t i = 0; i < n_loads; ++i)
    STQ_HOST_CHECK(load_expert[i] >= 0 && load_expert[i] < b->n_experts && load_slot[i] >= 0 &&
                       load_slot[i] < b->n_slots,
                   STQ_ERR_INVALID_ARG);
  cudaStream_t s = stq_cuda_stream(stream);
  // one copy per matrix and expert
  for (int32_t i = 0; i < n_loads; ++i)
    for (int32_t m = 0; m < n_mats; ++m) {
      const size_t bytes = mat_bytes[m];
      const char* from = static_cast<const char*>(src[m]) + size_t(load_expert[i]) * bytes;
      char* to = static_cast<char*>(dst[m]) + size_t(load_slot[i]) * bytes;
      if (cudaMemcpyAsync(to, from, bytes, cudaMemcpyDefault, s) != cudaSuccess) return STQ_ERR_CUDA;
    }
  return STQ_OK;
}
