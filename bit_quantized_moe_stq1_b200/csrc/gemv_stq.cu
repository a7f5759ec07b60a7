// Single-matrix STQ1_0 GEMV: y[n, r] = sum_k W[r, k] x[n, k].
//
// One CTA = one 16-row tile; its K blocks are split across the CTA's four warps
// and the four partial tiles are summed through shared memory in a fixed order
// (deterministic).  Tokens are processed in chunks of eight (the mma N).

#include "gemv.cuh"

namespace {

__global__ void __launch_bounds__(128) stq1_gemv_kernel(const uint8_t* __restrict__ W, int64_t rows, int64_t K,
                                                         const uint16_t* __restrict__ x, int64_t n,
                                                         float* __restrict__ y) {
  __shared__ float red[4][4][32];
  stq_pdl_begin();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, g = lane >> 2, t = lane & 3;
  const int nb = int(K / 256);
  const int64_t tile = blockIdx.x;
  const uint32_t lut = stq::lut_entry(lane);
  const uint8_t* tb[1] = {W + tile * nb * stq::kTileBlockBytes};
  const int b0 = (nb * warp) / 4, b1 = (nb * (warp + 1)) / 4;
  for (int64_t c0 = 0; c0 < n; c0 += 8) {
    const int64_t tok = c0 + g;
    const uint16_t* xrow = tok < n ? x + tok * K : nullptr;
    float acc[1][4] = {{0.f, 0.f, 0.f, 0.f}};
    stq::stq_warp_gemv<1>(tb, b0, b1, xrow, lut, acc);
#pragma unroll
    for (int j = 0; j < 4; ++j) red[warp][j][lane] = acc[0][j];
    __syncthreads();
    if (warp == 0) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float v = ((red[0][j][lane] + red[1][j][lane]) + red[2][j][lane]) + red[3][j][lane];
        const int64_t col = c0 + 2 * t + (j & 1);
        const int64_t row = tile * 16 + g + 8 * (j >> 1);
        if (col < n) y[col * rows + row] = v;
      }
    }
    __syncthreads();
  }
}

}  // namespace

extern "C" stq_status stq1_gemv(const uint8_t* W, int64_t rows, int64_t K, const uint16_t* x, int64_t n, float* y,
                                stq_stream_t stream) {
  STQ_HOST_CHECK(rows >= 0 && K >= 0 && n >= 0, STQ_ERR_INVALID_ARG);
  if (rows == 0 || n == 0) return STQ_OK;
  STQ_HOST_CHECK(W && x && y, STQ_ERR_INVALID_ARG);
  STQ_HOST_CHECK(rows % 16 == 0 && K % 256 == 0, STQ_ERR_SHAPE);
  STQ_HOST_CHECK(stq_aligned16(W) && stq_aligned16(x) && stq_aligned16(y), STQ_ERR_ALIGN);
  if (K == 0) return cudaMemsetAsync(y, 0, size_t(n * rows) * sizeof(float), stq_cuda_stream(stream)) == cudaSuccess
                         ? STQ_OK
                         : STQ_ERR_CUDA;
  {
    StqTimed tm(STQ_K_GEMV, stq_cuda_stream(stream));
    return stq_launch(stq1_gemv_kernel, dim3(unsigned(rows / 16)), dim3(128), 0, stq_cuda_stream(stream), W, rows, K, x,
                      n, y);
  }
}
