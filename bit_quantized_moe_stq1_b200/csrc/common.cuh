// Shared device/host helpers for the stqmoe kernels (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <stdint.h>

#include <mutex>
#include <utility>

#include "../../include/stqmoe.h"

#define STQ_HOST_CHECK(cond, code) \
  do {                             \
    if (!(cond)) return (code);    \
  } while (0)

static inline bool stq_aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static inline stq_status stq_launch_status() {
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? STQ_OK : STQ_ERR_CUDA;
}

static inline cudaStream_t stq_cuda_stream(stq_stream_t s) { return reinterpret_cast<cudaStream_t>(s); }

// Device ordinals covered by the library's per-device host caches.
constexpr int kStqMaxDevices = 64;

// Dynamic shared memory above 48 KB needs a per-kernel opt-in, and that attribute belongs
// to the kernel on one device.  One object per kernel records, per device, the size
// already allowed, so the driver call runs once per device and size.  Thread-safe.
struct StqSmemOptIn {
  std::mutex mu;
  int allowed[kStqMaxDevices] = {};

  template <typename Kernel>
  stq_status ensure(Kernel* kernel, int bytes) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kStqMaxDevices) return STQ_ERR_CUDA;
    std::lock_guard<std::mutex> lock(mu);
    if (allowed[dev] >= bytes) return STQ_OK;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
      return STQ_ERR_CUDA;
    allowed[dev] = bytes;
    return STQ_OK;
  }
};

// Programmatic dependent launch.  The hot-path kernels are launched with programmatic
// stream serialisation (stq_launch): a kernel may then start while its predecessor on the
// stream is still running.  Each one first lets its own successor launch, then waits until
// the predecessor has completed and its writes are visible, before it touches any global
// memory.  Launched without the attribute, both instructions do nothing.
__device__ __forceinline__ void stq_pdl_begin() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

// Launch with programmatic stream serialisation (see stq_pdl_begin).
template <typename... KArgs, typename... Args>
static inline stq_status stq_launch(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                                    Args&&... args) {
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr.val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...) == cudaSuccess ? STQ_OK : STQ_ERR_CUDA;
}

// First error wins: only replace a 0 word.
__device__ __forceinline__ void stq_set_error(int32_t* err, int32_t code) {
  if (err != nullptr) atomicCAS(err, 0, code);
}

// Checked build (-DSTQ_CHECKED=1, libstqmoe_checked.so): kernels re-check the indices they
// take from data (expert ids from the touched list, token indices from the permutation,
// sorted positions from the inverse map) before using them.  A failed check records
// STQ_ERR_DEVICE in the error word and the access is skipped; nothing traps.  In the
// default build STQ_DCHECK is the constant true and its condition is not evaluated.
#if defined(STQ_CHECKED) && STQ_CHECKED
__device__ __forceinline__ bool stq_dcheck(bool ok, int32_t* err) {
  if (!ok) stq_set_error(err, STQ_ERR_DEVICE);
  return ok;
}
#define STQ_DCHECK(cond, err) stq_dcheck((cond), (err))
#else
#define STQ_DCHECK(cond, err) true
#endif

__device__ __forceinline__ float bf16_bits_to_float(uint32_t b) { return __uint_as_float(b << 16); }

// float -> bf16 bits, round to nearest even (the library conversion intrinsic).
__device__ __forceinline__ uint16_t float_to_bf16_bits(float f) {
  __nv_bfloat16 h = __float2bfloat16_rn(f);
  return *reinterpret_cast<uint16_t*>(&h);
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// D = A * B + D for one m16n8k16 bf16 tile with FP32 accumulators.
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                               uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ float silu_f32(float g) { return g / (1.0f + expf(-g)); }

// 2^x as a float for x in [-127, 127] (2^-127 is the binary32 subnormal 0x00400000).
__device__ __forceinline__ float pow2_float(int x) {
  return x >= -126 ? __uint_as_float(uint32_t(x + 127) << 23) : __uint_as_float(0x00400000u);
}

// Biased UE8M0 exponent of the smallest power of two 2^k with amax <= limit * 2^k,
// where limit = 1.m * 2^p is given by its mantissa bits (m_lim) and exponent p
// (E4M3's 448 = 1.75 * 2^8: m_lim 0x600000, p 8; E2M1's 6 = 1.5 * 2^2: 0x400000, 2).
__device__ __forceinline__ int mx_scale_exponent(float amax, uint32_t m_lim, int p) {
  if (amax == 0.f) return 127;
  const uint32_t ab = __float_as_uint(amax);
  const int eb = int(ab >> 23);
  if (eb == 0) return 0;  // subnormal amax: k + 127 < 0
  const int E = eb - 127;
  const int k = ((ab & 0x7FFFFFu) <= m_lim) ? E - p : E - p + 1;
  return min(max(k + 127, 0), 254);
}

// E4M3 code (round to nearest even, saturating) of v * f; a zero result keeps v's sign.
__device__ __forceinline__ uint32_t e4m3_code(float v, float f) {
  const __nv_fp8_storage_t c = __nv_cvt_float_to_fp8(v * f, __NV_SATFINITE, __NV_E4M3);
  uint32_t code = c;
  if ((code & 0x7Fu) == 0u) code = (__float_as_uint(v) >> 31) << 7;
  return code;
}

// Round an FP32 value to the bf16 grid and back (for intermediates stored as bf16).
__device__ __forceinline__ float round_bf16(float f) { return __bfloat162float(__float2bfloat16_rn(f)); }

// Timing hook (abi.cu): bracket one kernel launch with events when installed.
struct StqTimed {
  StqTimed(int kind, cudaStream_t s);
  ~StqTimed();
  cudaStream_t s;
  int slot;
  bool capturing;
};

template <typename T>
__host__ __device__ constexpr T ceil_div(T a, T b) { return (a + b - 1) / b; }

static inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
