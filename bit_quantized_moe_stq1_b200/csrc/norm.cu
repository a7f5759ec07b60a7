// RMS normalisation of bf16 rows: the glue between consecutive MoE layers of a stack.
//
// One CTA per row.  Pass 1 sums the squares of the row in FP64 (each thread its
// strided uint4 chunks in ascending order, then a fixed xor-shuffle tree and the eight
// warp partials in warp order, so the result does not depend on timing; FP64 holds the
// square of any bf16 value, so no row overflows); pass 2 reads the row again (from
// L1/L2: a 6144-wide row is 12 KB) and writes x * (1 / sqrt(ms + eps)), multiplied in
// FP64 and rounded to FP32 and then to bf16 (round to nearest even at both steps).
// In place is allowed: every element is read and written by the same thread, and
// pass 2 begins only after the whole CTA has finished pass 1.

#include "common.cuh"

namespace {

constexpr int kThreads = 256;

__global__ void __launch_bounds__(kThreads) rmsnorm_bf16_kernel(const uint16_t* x, int H, float eps, uint16_t* y) {
  __shared__ double part[kThreads / 32];
  __shared__ double s_scale;
  const int row = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  stq_pdl_begin();
  const uint4* xr = reinterpret_cast<const uint4*>(x + size_t(row) * H);
  uint4* yr = reinterpret_cast<uint4*>(y + size_t(row) * H);
  const int n8 = H / 8;
  double ss = 0.0;
  for (int i = tid; i < n8; i += kThreads) {
    const uint4 v = xr[i];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const double a = bf16_bits_to_float(w[j] & 0xFFFFu), b = bf16_bits_to_float(w[j] >> 16);
      ss = fma(a, a, ss);
      ss = fma(b, b, ss);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if (lane == 0) part[warp] = ss;
  __syncthreads();
  if (tid == 0) {
    double t = 0.0;
#pragma unroll
    for (int w = 0; w < kThreads / 32; ++w) t += part[w];
    s_scale = 1.0 / sqrt(t / double(H) + double(eps));
  }
  __syncthreads();
  const double r = s_scale;
  for (int i = tid; i < n8; i += kThreads) {
    const uint4 v = xr[i];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t o[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float a = __double2float_rn(double(bf16_bits_to_float(w[j] & 0xFFFFu)) * r);
      const float b = __double2float_rn(double(bf16_bits_to_float(w[j] >> 16)) * r);
      o[j] = uint32_t(float_to_bf16_bits(a)) | (uint32_t(float_to_bf16_bits(b)) << 16);
    }
    yr[i] = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

}  // namespace

extern "C" stq_status stq_rmsnorm_bf16(const uint16_t* x, int64_t T, int64_t H, float eps, uint16_t* y,
                                       stq_stream_t stream) {
  STQ_HOST_CHECK(T >= 0 && H > 0, STQ_ERR_INVALID_ARG);
  STQ_HOST_CHECK(H % 8 == 0 && H <= (int64_t(1) << 24), STQ_ERR_SHAPE);
  STQ_HOST_CHECK(T <= 0x7fffffff, STQ_ERR_SHAPE);
  STQ_HOST_CHECK(eps >= 0.f && eps < 3.0e38f, STQ_ERR_INVALID_ARG);  // also rejects NaN
  if (T == 0) return STQ_OK;
  STQ_HOST_CHECK(x != nullptr && y != nullptr, STQ_ERR_INVALID_ARG);
  STQ_HOST_CHECK(stq_aligned16(x) && stq_aligned16(y), STQ_ERR_ALIGN);
  const cudaStream_t s = stq_cuda_stream(stream);
  StqTimed tm(STQ_K_RMSNORM, s);
  return stq_launch(rmsnorm_bf16_kernel, dim3(unsigned(T)), dim3(kThreads), 0, s, x, int(H), eps, y);
}
