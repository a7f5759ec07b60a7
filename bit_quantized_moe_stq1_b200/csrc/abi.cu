// Status strings, version, error-word access and instrumentation of the C ABI.
#include <nvtx3/nvToolsExt.h>

#include "moe_internal.cuh"

extern "C" const char* stq_status_string(stq_status s) {
  switch (s) {
    case STQ_OK: return "STQ_OK";
    case STQ_ERR_INVALID_ARG: return "STQ_ERR_INVALID_ARG";
    case STQ_ERR_SHAPE: return "STQ_ERR_SHAPE";
    case STQ_ERR_ALIGN: return "STQ_ERR_ALIGN";
    case STQ_ERR_NONFINITE: return "STQ_ERR_NONFINITE";
    case STQ_ERR_CUDA: return "STQ_ERR_CUDA";
    case STQ_ERR_DEVICE: return "STQ_ERR_DEVICE";
    case STQ_ERR_WORKSPACE: return "STQ_ERR_WORKSPACE";
    case STQ_ERR_TIMEOUT: return "STQ_ERR_TIMEOUT";
    case STQ_ERR_UNSUPPORTED: return "STQ_ERR_UNSUPPORTED";
    default: return "STQ_ERR_UNKNOWN";
  }
}

extern "C" int32_t stq_abi_version(void) { return STQMOE_ABI_VERSION; }

extern "C" int32_t stq_checked_build(void) {
#if defined(STQ_CHECKED) && STQ_CHECKED
  return 1;
#else
  return 0;
#endif
}

extern "C" stq_status stq_read_error(int32_t* err, stq_stream_t stream) {
  if (err == nullptr) return STQ_ERR_INVALID_ARG;
  cudaStream_t s = stq_cuda_stream(stream);
  int32_t host = 0;
  if (cudaMemcpyAsync(&host, err, sizeof(int32_t), cudaMemcpyDeviceToHost, s) != cudaSuccess) return STQ_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return STQ_ERR_CUDA;
  if (host != 0) {
    if (cudaMemsetAsync(err, 0, sizeof(int32_t), s) != cudaSuccess) return STQ_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return STQ_ERR_CUDA;
  }
  return host;
}

extern "C" stq_status moe_get_device_error(void* workspace, stq_stream_t stream) {
  if (workspace == nullptr) return STQ_ERR_INVALID_ARG;
  return stq_read_error(static_cast<int32_t*>(workspace), stream);
}

static stq_timing* g_timing = nullptr;

// Names of the STQ_K_* kernel kinds, in enum order.
static const char* const kKindNames[] = {"router_logits", "router_topk", "permute", "quant_x", "gate_up", "down",
                                         "combine", "gemv", "gemm", "gate_up_mx", "down_mx", "plan",
                                         "shared_gate_up", "shared_down", "rmsnorm", "pack_ls", "gate_up_stq_tc",
                                         "down_stq_tc", "act_limbs"};
static_assert(sizeof(kKindNames) / sizeof(kKindNames[0]) == STQ_K_COUNT, "one name per kernel kind");

extern "C" const char* stq_kernel_kind_name(int32_t kind) {
  return kind >= 0 && kind < STQ_K_COUNT ? kKindNames[kind] : "unknown";
}

extern "C" stq_status stq_set_timing(stq_timing* t) {
  g_timing = t;
  return STQ_OK;
}

static cudaError_t record(cudaEvent_t ev, cudaStream_t st, bool capturing) {
  // Inside stream capture the record becomes an event-record node of the graph.
  return capturing ? cudaEventRecordWithFlags(ev, st, cudaEventRecordExternal) : cudaEventRecord(ev, st);
}

StqTimed::StqTimed(int kind, cudaStream_t st) : s(st), slot(-1), capturing(false) {
  // an NVTX range per launch, named by kind (a no-op unless a profiler is attached)
  nvtxRangePushA(stq_kernel_kind_name(kind));
  stq_timing* t = g_timing;
  if (t == nullptr || t->count >= t->capacity) return;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(st, &cs) != cudaSuccess) return;
  capturing = cs == cudaStreamCaptureStatusActive;
  slot = t->count++;
  t->kinds[slot] = kind;
  record(static_cast<cudaEvent_t>(t->events[2 * slot]), st, capturing);
}

StqTimed::~StqTimed() {
  if (slot >= 0 && g_timing != nullptr)
    record(static_cast<cudaEvent_t>(g_timing->events[2 * slot + 1]), s, capturing);
  nvtxRangePop();
}
