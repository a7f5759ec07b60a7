// W4A8 (MXFP4 weights x MXFP8 activations) products.  Placeholder until the
// tcgen05 block-scaled grouped GEMM lands.
#include "moe_internal.cuh"

stq_status moe_mx_experts(const MoeArgs&, int, bool, cudaStream_t) { return STQ_ERR_UNSUPPORTED; }

extern "C" stq_status w4a8_gemm(const uint8_t* w_codes, const uint8_t* w_scales, int64_t N, int64_t K,
                                const uint8_t* a_codes, const uint8_t* a_scales, int64_t M, float* y, int32_t* err,
                                stq_stream_t stream) {
  (void)w_codes; (void)w_scales; (void)N; (void)K; (void)a_codes; (void)a_scales; (void)M; (void)y; (void)err;
  (void)stream;
  return STQ_ERR_UNSUPPORTED;
}
